"""Host-side tests of the C-ABI library: loading, exported symbols, the host
pattern expansion (bit-exact against the oracle's token-level scan and the
hand-derived counts) and argument validation. No GPU needed: every call here
returns before any CUDA work."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import attention_sink_long_b200 as lg
from attention_sink_long_b200 import build as lgbuild

from test_oracle import load_golden

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lg_attn.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    lgbuild.build()
    yield


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|lg_status_t|int32_t)\s+(lg_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol():
    names = header_functions()
    assert len(names) >= 14
    L = ctypes.CDLL(lgbuild.LIB)
    for n in names:
        assert hasattr(L, n), n
    assert sorted(lg.EXPORTED_SYMBOLS) == names


def test_strerror_and_version():
    assert lg.lg_strerror(0) == "ok"
    assert "workspace" in lg.lg_strerror(3)
    assert lg.lg_version() >= (1 << 16)


PATTERNS = [
    lg.Pattern(64, 1, 4, 0), lg.Pattern(64, 1, 16, 32), lg.Pattern(64, 0, 1, 0), lg.Pattern(64, 0, 1, 3),
    lg.Pattern(64, 3, 2, 5), lg.Pattern(64, 0, 7, 0), lg.Pattern.full(64), lg.Pattern(64, 100, 1, 0),
    lg.Pattern(16, 2, 3, 4), lg.Pattern(8, 1, 1, 1),
]


@pytest.mark.parametrize("p", PATTERNS)
@pytest.mark.parametrize("S_blocks", [1, 2, 7, 33])
def test_host_expansion_bit_exact_vs_oracle(p, S_blocks):
    S = p.block_size * S_blocks
    op = oracle.Pattern(*p)
    row_ptr, col = lg.lg_pattern_expand(p, S)
    o_ptr, o_col = oracle.block_lists(S, op)
    np.testing.assert_array_equal(row_ptr, o_ptr)
    np.testing.assert_array_equal(col, o_col)
    col_ptr, row = lg.lg_pattern_expand_t(p, S)
    t_ptr, t_row = oracle.block_lists_t(S, op)
    np.testing.assert_array_equal(col_ptr, t_ptr)
    np.testing.assert_array_equal(row, t_row)
    assert lg.lg_pattern_pairs(p, S) == oracle.pair_count(S, op)


@pytest.mark.parametrize("name", ["c1_sink_local4", "c2_sink_window", "c2_dense", "c3_block_sparse",
                                  "c3_analog_4096", "c4_sink_window"])
def test_host_counts_match_hand_counts(name):
    S, p, nnz, pairs = load_golden()[name]
    lp = lg.Pattern(p.block_size, p.sink_blocks, p.local_blocks, p.stride)
    row_ptr, col = lg.lg_pattern_expand(lp, S)
    assert int(row_ptr[-1]) == nnz
    assert np.all(np.diff(row_ptr) > 0)
    assert lg.lg_pattern_pairs(lp, S) == pairs
    col_ptr, row = lg.lg_pattern_expand_t(lp, S)
    assert int(col_ptr[-1]) == nnz


def test_expansion_capacity_idiom():
    L = lg.lib()
    p = lg._lg_pattern_t(64, 1, 4, 0)
    nnz = ctypes.c_int64(0)
    assert L.lg_pattern_expand(ctypes.byref(p), 1024, None, None, 0, ctypes.byref(nnz)) == 0
    assert nnz.value == 70
    rp = (ctypes.c_int32 * 17)()
    col = (ctypes.c_int32 * 10)()
    assert L.lg_pattern_expand(ctypes.byref(p), 1024, rp, col, 10, ctypes.byref(nnz)) == 6  # LG_ERR_CAPACITY
    assert L.lg_pattern_expand(ctypes.byref(p), 1000, rp, col, 10, ctypes.byref(nnz)) == 1  # not a multiple


def _fwd(**kw):
    L = lg.lib()
    a = dict(p=lg._lg_pattern_t(64, 1, 4, 0), q=0x10000, k=0x20000, v=0x30000, o=0x40000, lse=0x50000,
             B=1, S=1024, H=4, Hkv=4, D=64, scale=0.125)
    a.update(kw)
    p = a["p"]
    return L.lg_sparse_attn_fwd(None if p is None else ctypes.byref(p), a["q"], a["k"], a["v"], a["o"],
                                a.get("odt", 0), a["lse"], a["B"], a["S"], a["H"], a["Hkv"], a["D"], a["scale"],
                                None, 0, None)


def test_fwd_argument_errors():
    assert _fwd(p=None) == 1
    assert _fwd(q=None) == 1
    assert _fwd(B=0) == 1
    assert _fwd(H=4, Hkv=3) == 1
    assert _fwd(scale=0.0) == 1
    assert _fwd(scale=float("nan")) == 1
    assert _fwd(p=lg._lg_pattern_t(64, 1, 0, 0)) == 1      # local_blocks < 1
    assert _fwd(p=lg._lg_pattern_t(64, -1, 1, 0)) == 1     # negative sink
    assert _fwd(p=lg._lg_pattern_t(32, 1, 4, 0)) == 2      # block size other than 64
    assert _fwd(S=1000) == 2                               # S not a multiple of 64
    assert _fwd(D=96) == 2
    assert _fwd(q=0x10008) == 2                            # misaligned
    assert _fwd(lse=0x50004) == 2
    assert _fwd(odt=2) == 1                                # O dtype


def test_bwd_and_decode_argument_errors():
    L = lg.lib()
    p = lg._lg_pattern_t(64, 1, 4, 0)
    P = [0x10000 * (i + 1) for i in range(9)]

    def bwd(ptrs, odt=0, gdt=0, D=64, ws=None, wsb=0):
        return L.lg_sparse_attn_bwd(ctypes.byref(p), *ptrs[:4], odt, *ptrs[4:], gdt, 1, 1024, 4, 4, D, 0.125, ws,
                                    wsb, None)

    assert bwd(P) == 3                                  # workspace missing
    assert bwd(P, D=128, ws=0x100000, wsb=16) == 3      # workspace too small
    assert bwd([None] + P[1:]) == 1
    assert bwd(P, gdt=2) == 1                           # gradient dtype
    assert bwd(P, odt=5) == 1                           # O dtype
    args = [0x10000, 0x20000, 0x30000, 0x40000, 0x50000]  # q, k_cache, v_cache, cache_lens, o

    def dec(B=32, H=32, Hkv=32, D=128, L=4160, odt=0, lse=0x60000):
        return L_.lg_sparse_decode(*args, odt, lse, B, H, Hkv, D, L, 0, 0.1, None, 0, None)

    L_ = L
    assert dec(D=96) == 2                 # D
    assert dec(H=24, Hkv=8) == 2          # G = 3
    assert dec() == 3                     # workspace needed
    assert dec(L=0) == 1
    assert dec(odt=2) == 1                # o dtype
    assert dec(lse=0x60002) == 2          # misaligned lse


def test_workspace_queries():
    assert lg.lg_sparse_attn_fwd_workspace(lg.Pattern(64, 1, 64, 0), 1, 131072, 32, 32, 128) == 0
    ws = lg.lg_sparse_attn_bwd_workspace(lg.Pattern(64, 1, 64, 0), 1, 131072, 32, 32, 128)
    assert ws >= 131072 * 32 * 128 * 4 + 131072 * 32 * 4
    assert lg.lg_sparse_decode_splits(32, 32, 32, 128, 4160) > 1
    assert lg.lg_sparse_decode_splits(1, 1, 1, 128, 64, 1) == 1
    assert lg.lg_sparse_decode_workspace(1, 1, 1, 128, 64, 1) == 0
    ns = lg.lg_sparse_decode_splits(32, 32, 32, 128, 131072)
    assert lg.lg_sparse_decode_workspace(32, 32, 32, 128, 131072) >= 32 * 32 * ns * 129 * 4
    assert lg.lg_sparse_decode_splits(2, 8, 8, 128, 100, 7) == 7


def _r256(n):
    return (n + 255) // 256 * 256


def test_bwd_workspace_holds_split_sink_tile_partials():
    """32K sink+window: the other KV tiles walk ~33 query steps (66 blocks), the
    sink tile all 256, so its walk is split into ceil(256 / 33) = 8 chunks
    whose fp32 dV / dK partials (2 x 128 x D each, per KV head) and one counter
    per KV head join the workspace. Dense causal (no tile stands out) and the
    block-sparse pattern (several heavy tiles per head) keep the base size."""
    B, S, H, Hkv, D = 1, 32768, 32, 32, 128
    base = _r256(B * H * S * D * 4) + 2 * _r256(B * H * S * 4)
    ws = lg.lg_sparse_attn_bwd_workspace(lg.Pattern(64, 1, 64, 0), B, S, H, Hkv, D)
    assert ws == base + _r256(B * Hkv * 8 * 2 * 128 * D * 4) + _r256(B * Hkv * 4)
    assert lg.lg_sparse_attn_bwd_workspace(lg.Pattern.full(64), B, S, H, Hkv, D) == base
    assert lg.lg_sparse_attn_bwd_workspace(lg.Pattern(64, 1, 16, 32), B, S, H, Hkv, D) == base
    # short sequences: the sink tile's walk is no longer than one chunk, nothing is split
    assert lg.lg_sparse_attn_bwd_workspace(lg.Pattern(64, 1, 4, 0), 1, 1024, 4, 4, 64) == \
        _r256(1024 * 4 * 64 * 4) + 2 * _r256(4 * 1024 * 4)


@pytest.mark.parametrize("shape,splits", [
    # one query head per KV head: 512-row pieces, halved while B * Hkv * splits < 1184
    ((32, 32, 32, 128, 4160), 9), ((1, 32, 32, 128, 4160), 65), ((32, 32, 32, 64, 4160), 5),
    # query-head groups, more than 128 (b, kv head) pairs: ~1024-row pieces
    ((32, 32, 8, 128, 4160), 5), ((32, 32, 8, 128, 65536), 64), ((128, 32, 8, 128, 4160), 5),
    # at most 128 pairs: about 256 CTAs, never more pieces than 64-row blocks
    ((32, 32, 4, 128, 4160), 2), ((8, 32, 8, 128, 4160), 4), ((8, 32, 4, 128, 4160), 8),
    ((1, 32, 8, 128, 4160), 32), ((1, 8, 1, 128, 100), 2), ((1, 8, 1, 128, 64), 1),
])
def test_decode_split_rule(shape, splits):
    """The automatic split count the header documents (host logic only)."""
    B, H, Hkv, D, L = shape
    ns = lg.lg_sparse_decode_splits(B, H, Hkv, D, L)
    assert ns == splits
    rps = -(-L // ns)
    assert -(-L // rps) == ns and ns <= -(-L // 64)  # equal pieces cover the cache, none empty


# ---------------------------------------------------------------- prefill -> decode hand-off (host side)

@pytest.mark.parametrize("p", [(64, 1, 64, 0), (64, 1, 16, 32), (64, 0, 2**31 - 1, 0), (64, 0, 1, 0), (64, 1, 4, 0),
                               (64, 4, 8, 0), (64, 0, 2, 3), (64, 2, 3, 5), (64, 7, 1, 2), (64, 100, 1, 0)])
@pytest.mark.parametrize("S", [64, 128, 1024, 4096, 8192])
def test_compact_rows_match_oracle(p, S):
    """Host row count of the reduced cache equals the oracle's row list length, bit for bit."""
    assert lg.lg_kv_compact_rows(p, S) == len(oracle.reduced_cache_rows(S, oracle.Pattern(*p)))


def test_compact_argument_errors():
    L = lg.lib()
    p = lg._lg_pattern_t(64, 1, 64, 0)
    n = ctypes.c_int32(0)
    assert L.lg_kv_compact_rows(ctypes.byref(p), 1000, ctypes.byref(n)) == 2            # S % 64
    assert L.lg_kv_compact_rows(ctypes.byref(p), 0, ctypes.byref(n)) == 1
    assert L.lg_kv_compact_rows(ctypes.byref(p), 4096, None) == 1
    assert L.lg_kv_compact_rows(None, 4096, ctypes.byref(n)) == 1

    def compact(k=0x10000, v=0x20000, kc=0x30000, vc=0x40000, lens=0x50000, B=2, S=32768, Hkv=8, D=128, Lmax=4160):
        return L.lg_kv_compact(ctypes.byref(p), k, v, B, S, Hkv, D, kc, vc, Lmax, lens, None)

    assert compact(Lmax=4095) == 6          # 4096 rows do not fit
    assert compact(k=None) == 1
    assert compact(lens=None) == 1
    assert compact(B=0) == 1
    assert compact(D=96) == 2
    assert compact(S=1000) == 2
    assert compact(kc=0x30008) == 2         # misaligned


def test_fwd_varlen_argument_errors():
    L = lg.lib()
    p = lg._lg_pattern_t(64, 1, 4, 0)

    def call(q=0x10000, cu=0x60000, B=2, total=1024, mx=512, H=4, Hkv=4, D=128, odt=0, scale=0.125):
        return L.lg_sparse_attn_fwd_varlen(ctypes.byref(p), q, 0x20000, 0x30000, 0x40000, odt, 0x50000, cu, B,
                                           total, mx, H, Hkv, D, scale, None)

    assert call(q=None) == 1
    assert call(cu=None) == 1
    assert call(B=0) == 1
    assert call(H=4, Hkv=3) == 1
    assert call(odt=3) == 1
    assert call(scale=-1.0) == 1
    assert call(mx=500) == 2          # max_seqlen not a multiple of 64
    assert call(mx=2048) == 2         # longer than the packed tensor
    assert call(D=96) == 2
    assert call(q=0x10008) == 2       # misaligned
    assert call(cu=0x60002) == 2      # misaligned offsets


def test_wait_selftest_argument_errors():
    L = lg.lib()
    assert L.lg_wait_selftest(0, None) == 1
    assert L.lg_wait_selftest(5_000_000_000, None) == 1


def test_paged_cache_argument_errors():
    L = lg.lib()
    p = lg._lg_pattern_t(64, 1, 64, 0)

    def compact(k=0x10000, kp=0x30000, tbl=0x50000, ids=0x60000, lens=0x70000, pos=0x80000, B=2, S=32768, Hkv=8,
                D=128, P=256, MB=65, pat=p):
        return L.lg_kv_compact_paged(ctypes.byref(pat), k, 0x20000, B, S, Hkv, D, kp, 0x40000, P, tbl, ids, MB, lens,
                                     pos, None)

    assert compact(MB=63) == 6          # 64 blocks do not fit in 63 table entries
    assert compact(k=None) == 1
    assert compact(ids=None) == 1
    assert compact(pos=None) == 1
    assert compact(P=0) == 1
    assert compact(MB=0) == 1
    assert compact(S=1000) == 2
    assert compact(D=96) == 2
    assert compact(kp=0x30008) == 2     # misaligned pool
    assert compact(tbl=0x50002) == 2    # misaligned table
    assert compact(pat=lg._lg_pattern_t(32, 1, 64, 0)) == 2

    def append(kn=0x10000, kp=0x30000, tbl=0x50000, ids=0x60000, lens=0x70000, pos=0x80000, B=2, Hkv=8, D=128, P=256,
               MB=65):
        return L.lg_kv_append_paged(ctypes.byref(p), kn, 0x20000, B, Hkv, D, kp, 0x40000, P, tbl, ids, MB, lens, pos,
                                    None)

    assert append(kn=None) == 1
    assert append(tbl=None) == 1
    assert append(B=0) == 1
    assert append(MB=-1) == 1
    assert append(D=80) == 2
    assert append(kn=0x10004) == 2
    assert append(MB=(1 << 24) + 1) == 2

    def decode(q=0x10000, kp=0x30000, tbl=0x50000, lens=0x70000, B=2, H=8, Hkv=8, D=128, P=256, MB=65, ns=1,
               scale=0.088, ws=None, wsb=0, odt=0):
        return L.lg_sparse_decode_paged(q, kp, 0x40000, P, tbl, MB, lens, 0x90000, odt, None, B, H, Hkv, D, ns, scale,
                                        ws, wsb, None)

    assert decode(q=None) == 1
    assert decode(lens=None) == 1
    assert decode(P=0) == 1
    assert decode(MB=0) == 1
    assert decode(H=8, Hkv=3) == 1
    assert decode(scale=0.0) == 1
    assert decode(D=96) == 2
    assert decode(kp=0x30008) == 2
    assert decode(MB=(1 << 24) + 1) == 2
    assert decode(ns=4) == 3            # four splits need a workspace
    assert decode(odt=3) == 1           # o dtype


def test_bwd_varlen_argument_errors():
    L = lg.lib()
    p = lg._lg_pattern_t(64, 1, 4, 0)

    def call(q=0x10000, cu=0x60000, B=2, total=1024, mx=512, H=4, Hkv=4, D=128, odt=0, gdt=0, scale=0.125,
             ws=0x100000, wsb=1 << 30):
        return L.lg_sparse_attn_bwd_varlen(ctypes.byref(p), q, 0x20000, 0x30000, 0x40000, odt, 0x50000, 0x70000,
                                           0x80000, 0x90000, 0xa0000, gdt, cu, B, total, mx, H, Hkv, D, scale, ws, wsb,
                                           None)

    assert call(q=None) == 1
    assert call(cu=None) == 1
    assert call(B=0) == 1
    assert call(H=4, Hkv=3) == 1
    assert call(odt=3) == 1
    assert call(gdt=2) == 1
    assert call(scale=float("nan")) == 1
    assert call(mx=500) == 2          # max_seqlen not a multiple of 64
    assert call(mx=2048) == 2         # longer than the packed tensor
    assert call(total=1022) == 2      # LSE rows would not be 16-byte aligned
    assert call(D=96) == 2
    assert call(q=0x10008) == 2       # misaligned
    assert call(cu=0x60002) == 2      # misaligned offsets
    assert call(ws=None) == 3
    assert call(wsb=1024) == 3
    assert call(ws=0x100080) == 2     # workspace not 256-byte aligned


def test_fwd_fp8qk_argument_errors():
    L = lg.lib()
    p = lg._lg_pattern_t(64, 1, 64, 0)

    def call(q=0x10000, qd=1.0, kd=1.0, B=1, S=1024, H=4, Hkv=4, D=128, odt=0, scale=0.088):
        return L.lg_sparse_attn_fwd_fp8qk(ctypes.byref(p), q, 0x20000, 0x30000, qd, kd, 0x40000, odt, 0x50000, B, S,
                                          H, Hkv, D, scale, None)

    assert call(q=None) == 1
    assert call(qd=0.0) == 1
    assert call(kd=-2.0) == 1
    assert call(qd=float("inf")) == 1
    assert call(odt=5) == 1
    assert call(D=64) == 2            # fp8 Q/K: head dim 128 only
    assert call(S=1000) == 2
    assert call(q=0x10008) == 2


def test_fwd_pair_argument_errors():
    L = lg.lib()
    p = lg._lg_pattern_t(64, 1, 64, 0)

    def call(q=0x10000, B=1, S=1024, H=4, Hkv=4, D=128, odt=0, scale=0.088, lse=0x50000):
        return L.lg_sparse_attn_fwd_pair(ctypes.byref(p), q, 0x20000, 0x30000, 0x40000, odt, lse, B, S, H, Hkv, D,
                                         scale, None)

    assert call(q=None) == 1
    assert call(odt=5) == 1
    assert call(scale=0.0) == 1
    assert call(H=4, Hkv=3) == 1
    assert call(D=64) == 2            # the pair kernel: head dim 128 only
    assert call(S=1000) == 2
    assert call(q=0x10008) == 2
    assert call(lse=0x50004) == 2
