"""Variable-length prefill forward (lg_sparse_attn_fwd_varlen) through the
C-ABI vs the fp64 oracle, one sequence at a time (the pattern applies inside
each sequence, positions counted from its first row).

Also: equal-length sequences give bit-for-bit the fixed-length call's O and
LSE (the same kernel arithmetic); rows outside every sequence are left as
they were; an offset list that breaks the rules is reported through
lg_device_status (bit 4) while the valid sequences are still computed.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import attention_sink_long_b200 as lg
import synthetic_inputs as si
from parity import assert_close, LSE_TOL

pytestmark = pytest.mark.gpu

SENTINEL = -12345


def packed_inputs(lens, H, Hkv, D, seed=0):
    total = int(sum(lens))
    q, k, v = si.prefill_inputs(1, total, H, Hkv, D, seed=si.SEED_BASE + 100 + seed)
    return q[0], k[0], v[0]


def run_varlen(pat, q, k, v, cu, max_len, scale, odt=torch.bfloat16):
    total, H, D = q.shape
    o = torch.full((total, H, D), SENTINEL, dtype=torch.int16, device="cuda")
    o = o.view(torch.bfloat16) if odt == torch.bfloat16 else torch.full((total, H, D), float("nan"), device="cuda")
    lse = torch.full((H, total), float("nan"), dtype=torch.float32, device="cuda")
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    lg.lg_sparse_attn_fwd_varlen(pat, q.cuda(), k.cuda(), v.cuda(), o, lse, cu_d, max_len, scale)
    torch.cuda.synchronize()
    return o, lse


CASES = [
    # lens, H, Hkv, D, pattern, O dtype
    ([192, 64, 512, 1024, 320], 4, 2, 128, (64, 1, 4, 0), torch.float32),
    ([256, 640, 128], 2, 2, 128, (64, 1, 2, 4), torch.float32),
    ([384, 64, 448], 2, 1, 64, (64, 0, 2**31 - 1, 0), torch.float32),
    ([1024, 512], 4, 4, 128, (64, 1, 4, 0), torch.bfloat16),
]


@pytest.mark.parametrize("lens,H,Hkv,D,pat,odt", CASES)
def test_varlen_matches_oracle_per_sequence(lens, H, Hkv, D, pat, odt):
    q, k, v = packed_inputs(lens, H, Hkv, D)
    cu = [0] + list(np.cumsum(lens))
    scale = 1.0 / math.sqrt(D)
    o, lse = run_varlen(pat, q, k, v, cu, max(lens), scale, odt)
    assert lg.lg_device_status(0) == 0
    p = oracle.Pattern(*pat)
    for b, n in enumerate(lens):
        s0, s1 = cu[b], cu[b + 1]
        ro, rl = oracle.attention_forward(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], p, scale)
        assert_close(f"O seq{b}", o[s0:s1].float().cpu().numpy(), ro[0])
        got_l = lse[:, s0:s1].cpu().numpy()
        assert np.max(np.abs(got_l - rl[0])) <= LSE_TOL, (b, np.max(np.abs(got_l - rl[0])))


def test_equal_lengths_match_the_fixed_length_call_bitwise():
    B, S, H, Hkv, D = 3, 768, 4, 2, 128
    pat = (64, 1, 4, 0)
    scale = 1.0 / math.sqrt(D)
    q, k, v = si.prefill_inputs(B, S, H, Hkv, D)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty(B, S, H, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
    lg.lg_sparse_attn_fwd(pat, qd, kd, vd, o, lse, scale)
    ov, lv = run_varlen(pat, q.reshape(B * S, H, D), k.reshape(B * S, Hkv, D), v.reshape(B * S, Hkv, D),
                        [b * S for b in range(B + 1)], S, scale)
    assert torch.equal(ov.view(B, S, H, D).view(torch.int16), o.view(torch.int16))
    assert torch.equal(lv.view(H, B, S).permute(1, 0, 2), lse)


def test_rows_outside_every_sequence_are_not_written():
    lens, H, Hkv, D = [128, 256], 2, 2, 128
    q, k, v = packed_inputs([64] + lens + [64], H, Hkv, D, seed=1)
    cu = [64, 64 + 128, 64 + 128 + 256]  # rows [0, 64) and the last 64 rows belong to no sequence
    o, lse = run_varlen((64, 1, 2, 0), q, k, v, cu, 256, 0.125)
    assert lg.lg_device_status(0) == 0
    total = q.shape[0]
    assert torch.all(o[:64].view(torch.int16) == SENTINEL)
    assert torch.all(o[total - 64:].view(torch.int16) == SENTINEL)
    assert torch.all(torch.isnan(lse[:, :64])) and torch.all(torch.isnan(lse[:, total - 64:]))
    assert not torch.any(o[64:total - 64].view(torch.int16) == SENTINEL)


def test_bad_offsets_are_reported_and_skipped():
    lens, H, Hkv, D = [128, 192, 256], 2, 2, 128
    q, k, v = packed_inputs(lens, H, Hkv, D, seed=2)
    cu = [0, 128, 128 + 100, 128 + 192 + 256]  # sequence 1 has 100 rows: not a multiple of 64
    scale = 0.125
    o, lse = run_varlen((64, 1, 2, 0), q, k, v, cu, 448, scale)
    assert lg.lg_device_status(0) & 16
    assert lg.lg_device_status(0) == 0  # read and cleared
    p = oracle.Pattern(64, 1, 2, 0)
    ro, _ = oracle.attention_forward(q[None, :128], k[None, :128], v[None, :128], p, scale)
    assert_close("O seq0", o[:128].float().cpu().numpy(), ro[0])
    assert torch.all(o[128:228].view(torch.int16) == SENTINEL)  # the skipped sequence


# ---------------------------------------------------------------- backward
def run_varlen_fwd_bwd(pat, q, k, v, do, cu, max_len, scale, odt=torch.float32, gdt=torch.float32,
                       dq_fill=float("nan")):
    total, H, D = q.shape
    Hkv = k.shape[1]
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    o = torch.zeros(total, H, D, dtype=odt, device="cuda")
    lse = torch.zeros(H, total, dtype=torch.float32, device="cuda")
    lg.lg_sparse_attn_fwd_varlen(pat, qd, kd, vd, o, lse, cu_d, max_len, scale)
    dq = torch.full((total, H, D), dq_fill, dtype=gdt, device="cuda")
    dk = torch.full((total, Hkv, D), SENTINEL, dtype=torch.int16, device="cuda")
    dv = torch.full((total, Hkv, D), SENTINEL, dtype=torch.int16, device="cuda")
    if gdt == torch.float32:
        dk = torch.full((total, Hkv, D), float("nan"), device="cuda")
        dv = torch.full((total, Hkv, D), float("nan"), device="cuda")
    else:
        dk, dv = dk.view(torch.bfloat16), dv.view(torch.bfloat16)
    ws = torch.full((lg.lg_sparse_attn_bwd_workspace(pat, 1, total, H, Hkv, D),), 0xFF, dtype=torch.uint8,
                    device="cuda")
    lg.lg_sparse_attn_bwd_varlen(pat, qd, kd, vd, o, dod, lse, dq, dk, dv, cu_d, max_len, scale, ws)
    torch.cuda.synchronize()
    return dq, dk, dv


BWD_CASES = [
    # lens, H, Hkv, D, pattern, O dtype: head dims 128 and 64, with and without query-head groups
    ([192, 64, 512, 1024, 320], 2, 2, 128, (64, 1, 4, 0), torch.float32),
    ([256, 640, 128], 2, 2, 128, (64, 1, 2, 4), torch.float32),
    ([384, 64, 448], 4, 2, 128, (64, 0, 2, 3), torch.float32),
    ([320, 192, 576], 2, 1, 64, (64, 0, 2**31 - 1, 0), torch.float32),
    ([192, 64, 512, 1024, 320], 2, 2, 64, (64, 1, 4, 0), torch.float32),
    ([1024, 512], 2, 2, 128, (64, 1, 4, 0), torch.bfloat16),
]


@pytest.mark.parametrize("lens,H,Hkv,D,pat,odt", BWD_CASES)
def test_varlen_bwd_matches_oracle_per_sequence(lens, H, Hkv, D, pat, odt):
    total = int(sum(lens))
    q, k, v, do = si.prefill_inputs(1, total, H, Hkv, D, seed=si.SEED_BASE + 110, with_dout=True)
    q, k, v, do = q[0], k[0], v[0], do[0]
    cu = [0] + list(np.cumsum(lens))
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = run_varlen_fwd_bwd(pat, q, k, v, do, cu, max(lens), scale, odt)
    assert lg.lg_device_status(0) == 0
    p = oracle.Pattern(*pat)
    for b in range(len(lens)):
        s0, s1 = cu[b], cu[b + 1]
        rdq, rdk, rdv, _ = oracle.attention_backward(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1],
                                                     do[None, s0:s1], p, scale)
        assert_close(f"dQ seq{b}", dq[s0:s1].cpu().numpy(), rdq[0])
        assert_close(f"dK seq{b}", dk[s0:s1].cpu().numpy(), rdk[0])
        assert_close(f"dV seq{b}", dv[s0:s1].cpu().numpy(), rdv[0])


@pytest.mark.parametrize("H,Hkv,D", [(4, 4, 128), (4, 2, 64)])
def test_varlen_bwd_equal_lengths_match_the_fixed_length_call(H, Hkv, D):
    """dK / dV bit for bit (each written by one CTA: at 768 rows the
    fixed-length call does not split the sink tile's walk either); dQ to
    within the order of its reduce-adds."""
    B, S = 3, 768
    pat = (64, 1, 4, 0)
    scale = 1.0 / math.sqrt(D)
    q, k, v, do = si.prefill_inputs(B, S, H, Hkv, D, with_dout=True)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o = torch.empty(B, S, H, D, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
    lg.lg_sparse_attn_fwd(pat, qd, kd, vd, o, lse, scale)
    dq = torch.empty(B, S, H, D, device="cuda")
    dk = torch.empty(B, S, Hkv, D, device="cuda")
    dv = torch.empty_like(dk)
    ws = torch.empty(lg.lg_sparse_attn_bwd_workspace(pat, B, S, H, Hkv, D), dtype=torch.uint8, device="cuda")
    lg.lg_sparse_attn_bwd(pat, qd, kd, vd, o, dod, lse, dq, dk, dv, scale, ws)
    flat = lambda t: t.reshape(B * S, *t.shape[2:])  # noqa: E731
    vdq, vdk, vdv = run_varlen_fwd_bwd(pat, flat(q), flat(k), flat(v), flat(do), [b * S for b in range(B + 1)], S,
                                       scale)
    assert lg.lg_device_status(0) == 0
    assert torch.equal(vdk, flat(dk)) and torch.equal(vdv, flat(dv))
    assert torch.allclose(vdq, flat(dq), rtol=1e-5, atol=1e-5)


def test_varlen_bwd_rows_outside_every_sequence():
    lens, H, Hkv, D = [128, 256], 2, 2, 128
    total = 64 + 128 + 256 + 64
    q, k, v, do = si.prefill_inputs(1, total, H, Hkv, D, seed=si.SEED_BASE + 111, with_dout=True)
    q, k, v, do = q[0], k[0], v[0], do[0]
    cu = [64, 64 + 128, 64 + 128 + 256]
    pat = (64, 1, 2, 0)
    dq, dk, dv = run_varlen_fwd_bwd(pat, q, k, v, do, cu, 256, 0.125, gdt=torch.bfloat16, dq_fill=7.0)
    assert lg.lg_device_status(0) == 0
    for t in (dk, dv):
        assert torch.all(t[:64].view(torch.int16) == SENTINEL)
        assert torch.all(t[total - 64:].view(torch.int16) == SENTINEL)
        assert not torch.any(t[64:total - 64].view(torch.int16) == SENTINEL)
    assert torch.all(dq[:64] == 0) and torch.all(dq[total - 64:] == 0)
    # The bf16 gradients are the fp32 ones rounded (the fp32 run is checked against the oracle above).
    fq, fk, fv = run_varlen_fwd_bwd(pat, q, k, v, do, cu, 256, 0.125)
    for name, g, f in (("dK", dk, fk), ("dV", dv, fv)):
        r = f[64:total - 64].to(torch.bfloat16).float()
        ulp = torch.where(r == 0, torch.full_like(r, 2.0 ** -133), torch.abs(r) * 2.0 ** -7)
        assert (torch.abs(g[64:total - 64].float() - r) > ulp * 1.0001).sum().item() == 0, name


def test_varlen_bwd_bad_offsets_are_reported_and_skipped():
    lens, H, Hkv, D = [128, 192, 256], 2, 2, 128
    total = sum(lens)
    q, k, v, do = si.prefill_inputs(1, total, H, Hkv, D, seed=si.SEED_BASE + 112, with_dout=True)
    q, k, v, do = q[0], k[0], v[0], do[0]
    cu = [0, 128, 128 + 100, total]  # sequence 1 has 100 rows: not a multiple of 64
    dq, dk, dv = run_varlen_fwd_bwd((64, 1, 2, 0), q, k, v, do, cu, 256, 0.125)
    st = lg.lg_device_status(0)
    assert st & 16, st
    assert lg.lg_device_status(0) == 0
    rdq, rdk, rdv, _ = oracle.attention_backward(q[None, :128], k[None, :128], v[None, :128], do[None, :128],
                                                 oracle.Pattern(64, 1, 2, 0), 0.125)
    assert_close("dK seq0", dk[:128].cpu().numpy(), rdk[0])
    assert torch.all(torch.isnan(dk[128:228]))  # the skipped sequence's rows are not written


def test_varlen_bench_workload_sampled():
    """The packed workload bench.py times (8 sink+window sequences of 32K..512
    tokens, H32 D128, bf16 O as in training): O rows, dQ rows and dK / dV rows
    of sampled blocks of the first, a middle and the last sequence vs the
    oracle run on that sequence alone."""
    lens = [32768, 16384, 8192, 4096, 2048, 1024, 512, 512]
    H, D = 32, 128
    pat = (64, 1, 64, 0)
    op = oracle.Pattern(*pat)
    total = sum(lens)
    cu = [0] + list(np.cumsum(lens))
    dev = torch.device("cuda")
    q = si.device_normal((total, H, D), si.SEED_BASE + 0, dev)
    k = si.device_normal((total, H, D), si.SEED_BASE + 1, dev)
    v = si.device_normal((total, H, D), si.SEED_BASE + 2, dev)
    do = si.device_normal((total, H, D), si.SEED_BASE + 3, dev)
    scale = 1.0 / math.sqrt(D)
    cu_d = torch.tensor(cu, dtype=torch.int32, device=dev)
    o = torch.empty(total, H, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(H, total, dtype=torch.float32, device=dev)
    lg.lg_sparse_attn_fwd_varlen(pat, q, k, v, o, lse, cu_d, max(lens), scale)
    dq, dk, dv = (torch.empty(total, H, D, dtype=torch.float32, device=dev) for _ in range(3))
    ws = torch.empty(lg.lg_sparse_attn_bwd_workspace(pat, 1, total, H, H, D), dtype=torch.uint8, device=dev)
    lg.lg_sparse_attn_bwd_varlen(pat, q, k, v, o, do, lse, dq, dk, dv, cu_d, max(lens), scale, ws)
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0
    rng = np.random.default_rng(3)
    for b, h in ((0, 0), (3, 17), (7, H - 1)):
        s0, n = cu[b], lens[b]
        nqb = n // 64
        qh, kh, vh, doh = (t[s0:s0 + n, h].float().cpu().numpy() for t in (q, k, v, do))
        blocks = sorted({0, nqb - 1, *rng.choice(np.arange(nqb), min(nqb, 3), replace=False).tolist()})
        rows = np.concatenate([np.arange(i * 64, i * 64 + 64) for i in blocks])
        ro, rl = oracle.attention_rows(qh, kh, vh, rows, op, scale)
        assert_close(f"O seq{b} h{h}", o[s0 + rows, h].float().cpu().numpy(), ro)
        assert np.max(np.abs(lse[h, s0 + rows].cpu().numpy() - rl)) <= LSE_TOL
        rdq, _ = oracle.attention_backward_rows(qh, kh, vh, doh, rows, op, scale)
        assert_close(f"dQ seq{b} h{h}", dq[s0 + rows, h].cpu().numpy(), rdq)
        krows = np.concatenate([np.arange(j * 64, j * 64 + 64) for j in blocks[:3]])
        rdk, rdv = oracle.attention_backward_kv_rows(qh, kh, vh, doh, krows, op, scale, chunk=256)
        assert_close(f"dK seq{b} h{h}", dk[s0 + krows, h].cpu().numpy(), rdk)
        assert_close(f"dV seq{b} h{h}", dv[s0 + krows, h].cpu().numpy(), rdv)


def test_varlen_zero_length_sequence():
    """An empty sequence between two others: forward and backward leave it
    out, the others match the oracle."""
    lens, H, Hkv, D = [192, 0, 320], 2, 2, 128
    total = sum(lens)
    q, k, v, do = si.prefill_inputs(1, total, H, Hkv, D, seed=si.SEED_BASE + 113, with_dout=True)
    q, k, v, do = q[0], k[0], v[0], do[0]
    cu = [0, 192, 192, 512]
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = run_varlen_fwd_bwd((64, 1, 2, 0), q, k, v, do, cu, 320, scale)
    assert lg.lg_device_status(0) == 0
    p = oracle.Pattern(64, 1, 2, 0)
    for s0, s1 in ((0, 192), (192, 512)):
        rdq, rdk, rdv, _ = oracle.attention_backward(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1],
                                                     do[None, s0:s1], p, scale)
        assert_close(f"dQ {s0}", dq[s0:s1].cpu().numpy(), rdq[0])
        assert_close(f"dK {s0}", dk[s0:s1].cpu().numpy(), rdk[0])
        assert_close(f"dV {s0}", dv[s0:s1].cpu().numpy(), rdv[0])
