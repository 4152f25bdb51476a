"""Backward parity: the tcgen05 backward (preprocess, main, dQ convert) through
the C-ABI vs the fp64 oracle's analytic gradients.

O and LSE come from the library's own forward (they are inputs of the
backward); the oracle computes its gradients from Q, K, V and dO alone.
Parity is checked on the fp32 gradient outputs (the accumulators before any
output rounding), at max |err| <= 1e-2 and mean |err| <= 1e-3; the bf16
outputs are checked to be those fp32 values rounded to nearest even (within
one bf16 ulp, since the order of the dQ reduce-adds varies between runs).
The benchmark workloads (1K attention-sink, 128K sink+window and 128K
block-sparse) run the training configuration: bf16 O from the forward. The other shapes take the
forward's fp32 O, which makes Delta = rowsum(dO * O) exact to fp32: with a
bf16 O, Delta alone carries ~1e-3 relative error, which reaches the 1e-2
bound on dQ / dK for shapes with large gradients (GQA groups).
Small shapes are compared in full; the 128K training workloads on sampled
query blocks (dQ) and KV blocks (dK, dV -- the sink block gathers every query
of the sequence; with the strided pattern, block nqb/2 is a strided block).
"""

import math

import numpy as np
import pytest
import torch

import oracle
import attention_sink_long_b200 as lg
import synthetic_inputs as si
from parity import assert_close

pytestmark = pytest.mark.gpu


def run_fwd_bwd(pattern, q, k, v, do, scale, grad_dtype=torch.float32, o_dtype=torch.bfloat16):
    B, S, H, D = q.shape
    Hkv = k.shape[2]
    o = torch.empty(q.shape, dtype=o_dtype, device=q.device)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    lg.lg_sparse_attn_fwd(pattern, q, k, v, o, lse, scale)
    dq = torch.empty(q.shape, dtype=grad_dtype, device=q.device)
    dk = torch.empty(k.shape, dtype=grad_dtype, device=q.device)
    dv = torch.empty(v.shape, dtype=grad_dtype, device=q.device)
    ws = torch.empty(lg.lg_sparse_attn_bwd_workspace(pattern, B, S, H, Hkv, D), dtype=torch.uint8, device=q.device)
    ws.fill_(0xFF)  # poisoned: the backward must not depend on the workspace contents
    lg.lg_sparse_attn_bwd(pattern, q, k, v, o, do, lse, dq, dk, dv, scale, ws)
    torch.cuda.synchronize()
    assert lg.lg_device_status(q.device.index or 0) == 0
    return dq, dk, dv


def assert_bf16_rounding_of(name, got_bf16, ref_f32, atol=0.0):
    """got_bf16 equals ref_f32 rounded to bf16, within one bf16 ulp (plus atol,
    for dQ: its terms arrive through fp32 atomic adds in an order that varies
    between runs, so two runs' fp32 dQ differ by that rounding -- a few units
    of 2^-24 of the terms' size -- which near a cancellation to zero is more
    than a relative bf16 ulp; dK and dV are summed in a fixed order)."""
    r = ref_f32.to(torch.bfloat16).float()
    g = got_bf16.float()
    ulp = torch.where(r == 0, torch.full_like(r, 2.0 ** -133), torch.abs(r) * 2.0 ** -7)
    bad = (torch.abs(g - r) > ulp * 1.0001 + atol).sum().item()
    assert bad == 0, (name, bad)


SMALL = [
    # B, S, H, Hkv, D, pattern, O dtype
    (1, 1024, 4, 4, 64, lg.Pattern(64, 1, 4, 0), torch.bfloat16),   # the 1K attention-sink workload
    (1, 1024, 4, 4, 64, lg.Pattern(64, 1, 4, 0), torch.float32),
    (1, 192, 2, 2, 128, lg.Pattern(64, 1, 1, 0), torch.float32),    # ragged 64-row tail KV tile
    (2, 384, 4, 2, 128, lg.Pattern(64, 0, 2, 3), torch.float32),    # GQA, strided, no sink
    (1, 512, 2, 2, 64, lg.Pattern.full(64), torch.float32),         # dense causal
    (1, 640, 4, 1, 128, lg.Pattern(64, 2, 3, 0), torch.float32),    # 4 query heads per KV head
    (1, 64, 1, 1, 128, lg.Pattern(64, 1, 1, 0), torch.float32),     # a single block
    (1, 2048, 2, 2, 128, lg.Pattern(64, 1, 16, 4), torch.float32),
    (1, 1280, 2, 2, 128, lg.Pattern(64, 0, 1, 0), torch.float32),   # diagonal only
    (2, 640, 2, 2, 128, lg.Pattern.full(64), torch.float32),        # dense causal, odd 128-row step count
    (1, 1024, 2, 2, 128, lg.Pattern(64, 1, 4, 0), torch.bfloat16),  # attention sink at head dim 128, bf16 O
    (1, 512, 8, 1, 128, lg.Pattern(64, 1, 2, 0), torch.float32),    # 8 query heads per KV head
    # head dim 64 on the same 128-row-step kernel
    (1, 192, 2, 2, 64, lg.Pattern(64, 1, 1, 0), torch.float32),     # ragged 64-row tail KV tile
    (1, 64, 1, 1, 64, lg.Pattern(64, 1, 1, 0), torch.float32),      # a single block
    (1, 2048, 2, 2, 64, lg.Pattern(64, 1, 16, 4), torch.float32),   # sink + window + strided blocks
    (1, 1280, 2, 2, 64, lg.Pattern(64, 0, 1, 0), torch.float32),    # diagonal only
    (2, 640, 2, 2, 64, lg.Pattern.full(64), torch.bfloat16),        # dense causal, odd 128-row step count
    (1, 512, 8, 1, 64, lg.Pattern(64, 1, 2, 0), torch.float32),     # 8 query heads per KV head
    # The sink tile's walk split into chunks (32 and 48 query steps against a chunk of 16):
    # its dV / dK are summed from the chunks' partials.
    (1, 4096, 2, 2, 128, lg.Pattern(64, 1, 4, 0), torch.float32),
    (1, 6144, 4, 2, 64, lg.Pattern(64, 1, 2, 0), torch.float32),
    (2, 4096, 2, 2, 64, lg.Pattern(64, 1, 4, 0), torch.float32),    # two batch rows, each split
]


@pytest.mark.parametrize("B,S,H,Hkv,D,pat,odt", SMALL)
def test_bwd_matches_oracle_small(B, S, H, Hkv, D, pat, odt):
    q, k, v, do = si.prefill_inputs(B, S, H, Hkv, D, with_dout=True)
    scale = 1.0 / math.sqrt(D)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    dq, dk, dv = run_fwd_bwd(pat, qd, kd, vd, dod, scale, o_dtype=odt)
    rdq, rdk, rdv, _ = oracle.attention_backward(q, k, v, do, oracle.Pattern(*pat), scale)
    assert_close("dQ", dq.cpu().numpy(), rdq)
    assert_close("dK", dk.cpu().numpy(), rdk)
    assert_close("dV", dv.cpu().numpy(), rdv)
    bq, bk, bv = run_fwd_bwd(pat, qd, kd, vd, dod, scale, torch.bfloat16, o_dtype=odt)
    assert_bf16_rounding_of("dQ", bq, dq, atol=float(dq.abs().max()) * 2.0 ** -16)
    assert_bf16_rounding_of("dK", bk, dk)
    assert_bf16_rounding_of("dV", bv, dv)


GQA_TRAINING = [
    # B, S, H, Hkv, D, pattern -- query-head groups with the forward's bf16 O (the training format)
    (2, 384, 4, 2, 128, lg.Pattern(64, 0, 2, 3)),
    (1, 640, 4, 1, 128, lg.Pattern(64, 2, 3, 0)),
    (1, 512, 8, 1, 128, lg.Pattern(64, 1, 2, 0)),
    (1, 1024, 4, 1, 64, lg.Pattern(64, 1, 4, 0)),
    (2, 512, 4, 2, 64, lg.Pattern(64, 1, 2, 4)),
]


@pytest.mark.parametrize("B,S,H,Hkv,D,pat", GQA_TRAINING)
def test_bwd_gqa_training_format_small(B, S, H, Hkv, D, pat):
    """Query-head groups with the bf16 O the forward writes for training,
    compared in full. The backward forms Delta = rowsum(dO * O) from the O it
    is handed, so the reference is the oracle's gradient with Delta taken from
    that same bf16 O: the comparison then measures the kernel, not the bf16
    rounding of its O input (which alone moves dK by up to ~1e-2 on these
    shapes)."""
    q, k, v, do = si.prefill_inputs(B, S, H, Hkv, D, with_dout=True)
    scale = 1.0 / math.sqrt(D)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
    lg.lg_sparse_attn_fwd(pat, qd, kd, vd, o, lse, scale)
    ws = torch.empty(lg.lg_sparse_attn_bwd_workspace(pat, B, S, H, Hkv, D), dtype=torch.uint8, device="cuda")
    grads = {}
    for dt in (torch.float32, torch.bfloat16):
        g = tuple(torch.empty(t.shape, dtype=dt, device="cuda") for t in (qd, kd, vd))
        ws.fill_(0xFF)
        lg.lg_sparse_attn_bwd(pat, qd, kd, vd, o, dod, lse, *g, scale, ws)
        grads[dt] = g
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0
    rdq, rdk, rdv, _ = oracle.attention_backward(q, k, v, do, oracle.Pattern(*pat), scale, o=o.cpu())
    dq, dk, dv = grads[torch.float32]
    assert_close("dQ", dq.cpu().numpy(), rdq)
    assert_close("dK", dk.cpu().numpy(), rdk)
    assert_close("dV", dv.cpu().numpy(), rdv)
    for name, b16, f32 in zip(("dQ", "dK", "dV"), grads[torch.bfloat16], grads[torch.float32]):
        assert_bf16_rounding_of(name, b16, f32, atol=float(f32.abs().max()) * 2.0 ** -16 if name == "dQ" else 0.0)


@pytest.mark.parametrize("pat", [lg.Pattern(64, 1, 64, 0), lg.Pattern(64, 1, 16, 32)],
                         ids=["sink_window", "block_sparse"])
def test_bwd_128k_sampled(pat):
    B, S, H, D = 1, 131072, 32, 128
    op = oracle.Pattern(*pat)
    dev = torch.device("cuda")
    q, k, v, do = si.prefill_inputs_device(B, S, H, H, D, dev, with_dout=True)
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = run_fwd_bwd(pat, q, k, v, do, scale)
    nqb = S // 64
    rng = np.random.default_rng(7)
    qblocks = sorted({0, 1, nqb - 2, nqb - 1, *rng.choice(np.arange(2, nqb - 2), 6, replace=False).tolist()})
    qrows = np.concatenate([np.arange(i * 64, i * 64 + 64) for i in qblocks])
    for h, kvblocks in ((0, [0, 1, nqb // 2, nqb - 1]), (H - 1, [1, nqb // 2, nqb - 1])):
        qh, kh, vh, doh = (t[0, :, h].float().cpu().numpy() for t in (q, k, v, do))
        rdq, _ = oracle.attention_backward_rows(qh, kh, vh, doh, qrows, op, scale)
        assert_close(f"dQ h{h}", dq[0, qrows, h].cpu().numpy(), rdq)
        krows = np.concatenate([np.arange(j * 64, j * 64 + 64) for j in kvblocks])
        rdk, rdv = oracle.attention_backward_kv_rows(qh, kh, vh, doh, krows, op, scale, chunk=256)
        assert_close(f"dK h{h}", dk[0, krows, h].cpu().numpy(), rdk)
        assert_close(f"dV h{h}", dv[0, krows, h].cpu().numpy(), rdv)


def _gqa_sampled(S, H, Hkv, pat, qblocks, kvblocks, D=128):
    """O and dQ rows of sampled query blocks and dK / dV rows of sampled KV
    blocks against the oracle, which sums dK / dV over the query heads of the
    KV head (bf16 O as in training)."""
    B = 1
    op = oracle.Pattern(*pat)
    G = H // Hkv
    dev = torch.device("cuda")
    q, k, v, do = si.prefill_inputs_device(B, S, H, Hkv, D, dev, with_dout=True)
    scale = 1.0 / math.sqrt(D)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    lg.lg_sparse_attn_fwd(pat, q, k, v, o, lse, scale)
    dq, dk, dv = (torch.empty(t.shape, dtype=torch.float32, device=dev) for t in (q, k, v))
    ws = torch.empty(lg.lg_sparse_attn_bwd_workspace(pat, B, S, H, Hkv, D), dtype=torch.uint8, device=dev)
    lg.lg_sparse_attn_bwd(pat, q, k, v, o, do, lse, dq, dk, dv, scale, ws)
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0
    qrows = np.concatenate([np.arange(i * 64, i * 64 + 64) for i in qblocks])
    krows = np.concatenate([np.arange(j * 64, j * 64 + 64) for j in kvblocks])
    for kvh in (0, Hkv - 1):
        kh, vh = (t[0, :, kvh].float().cpu().numpy() for t in (k, v))
        rdk = np.zeros((len(krows), D))
        rdv = np.zeros((len(krows), D))
        for g in range(G):
            h = kvh * G + g
            qh, doh = (t[0, :, h].float().cpu().numpy() for t in (q, do))
            if g in (0, G - 1):
                ro, _ = oracle.attention_rows(qh, kh, vh, qrows, op, scale)
                assert_close(f"O h{h}", o[0, qrows, h].float().cpu().numpy(), ro)
                rdq, _ = oracle.attention_backward_rows(qh, kh, vh, doh, qrows, op, scale)
                assert_close(f"dQ h{h}", dq[0, qrows, h].cpu().numpy(), rdq)
            a, b = oracle.attention_backward_kv_rows(qh, kh, vh, doh, krows, op, scale, chunk=256)
            rdk += a
            rdv += b
        assert_close(f"dK kvh{kvh}", dk[0, krows, kvh].cpu().numpy(), rdk)
        assert_close(f"dV kvh{kvh}", dv[0, krows, kvh].cpu().numpy(), rdv)


def test_gqa_32k_sampled():
    """The grouped-query workload bench.py times: 32K sink+window, H32 Hkv8 D128."""
    nqb = 32768 // 64
    _gqa_sampled(32768, 32, 8, lg.Pattern(64, 1, 64, 0), (0, 7, nqb // 2, nqb - 1), (0, 1, nqb // 3, nqb - 1))


def test_gqa_64k_block_sparse_sampled():
    """64K block-sparse {64,1,16,32}, H8 Hkv2: a head has 17 heavy (sink /
    strided) KV tiles, which then run together and walk the query blocks from
    the end of the sequence downwards. Sampled: the sink and strided KV blocks
    (each a heavy tile), a window-only block, the last block."""
    nqb = 65536 // 64
    _gqa_sampled(65536, 8, 2, lg.Pattern(64, 1, 16, 32), (0, 33, nqb // 2 + 5, nqb - 1),
                 (0, 32, nqb // 2, nqb // 2 + 7, nqb - 1))


def test_d64_32k_sampled():
    """The head-dim-64 workload bench.py times: 32K sink+window, H32, D64."""
    nqb = 32768 // 64
    _gqa_sampled(32768, 32, 32, lg.Pattern(64, 1, 64, 0), (0, 5, nqb // 2, nqb - 1), (0, 1, nqb // 3, nqb - 1), D=64)


def test_bwd_split_sink_tile_is_deterministic():
    """The sink tile's dV / dK are summed from its chunks' partials in chunk
    order, whichever chunk finishes last: two runs give the same bits."""
    B, S, H, D = 1, 8192, 4, 128
    pat = lg.Pattern(64, 1, 16, 0)
    q, k, v, do = si.prefill_inputs(B, S, H, H, D, with_dout=True)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    a = run_fwd_bwd(pat, qd, kd, vd, dod, 1.0 / math.sqrt(D))
    b = run_fwd_bwd(pat, qd, kd, vd, dod, 1.0 / math.sqrt(D))
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
