"""Forward parity: the tcgen05 prefill kernel through the C-ABI vs the fp64 oracle.

Small shapes are compared element by element (several 128-row tiles, a ragged
64-row tail, GQA, every pattern term, D = 64 and 128). The CTA-pair forward
(lg_sparse_attn_fwd_pair, head dim 128) runs the same cases, including
512-row spans the sequence end cuts short, and two full-size workloads. The full-size workloads
(32K sink+window and dense, 128K block-sparse) are compared on sampled query
blocks of the first and last head, whose rows the oracle computes one by one.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import attention_sink_long_b200 as lg
import synthetic_inputs as si
from parity import assert_close, assert_lse

pytestmark = pytest.mark.gpu


def run_fwd(pattern, q, k, v, scale, o_dtype=torch.bfloat16):
    B, S, H, D = q.shape
    o = torch.empty(q.shape, dtype=o_dtype, device=q.device)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    lg.lg_sparse_attn_fwd(pattern, q, k, v, o, lse, scale)
    torch.cuda.synchronize()
    assert lg.lg_device_status(q.device.index or 0) == 0
    return o, lse


SMALL = [
    # B, S, H, Hkv, D, pattern
    (1, 1024, 4, 4, 64, lg.Pattern(64, 1, 4, 0)),      # the 1K attention-sink workload
    (1, 192, 2, 2, 128, lg.Pattern(64, 1, 1, 0)),      # ragged 64-row tail tile
    (2, 384, 4, 2, 128, lg.Pattern(64, 0, 2, 3)),      # GQA, strided, no sink
    (1, 512, 2, 2, 64, lg.Pattern.full(64)),           # dense causal
    (1, 640, 2, 1, 128, lg.Pattern(64, 2, 3, 0)),      # 2 query heads per KV head
    (1, 64, 1, 1, 128, lg.Pattern(64, 1, 1, 0)),       # a single block
    (1, 2048, 2, 2, 128, lg.Pattern(64, 1, 16, 4)),
    (1, 1280, 2, 2, 128, lg.Pattern(64, 0, 1, 0)),     # diagonal only: first block half-masked per tile
    (1, 1024, 2, 2, 128, lg.Pattern(64, 1, 2, 5)),
    # For the CTA-pair forward (512-row spans): spans cut short by the sequence end (one block
    # left: the odd CTA has no rows; 384 rows left: the odd CTA's second tile has none), and
    # unions of odd length (a lone last block in the chunk walk).
    (1, 576, 2, 2, 128, lg.Pattern(64, 1, 2, 0)),
    (2, 896, 4, 4, 128, lg.Pattern(64, 0, 3, 0)),
    (1, 1536, 4, 1, 128, lg.Pattern(64, 3, 2, 5)),
    # Head dim 64: ragged tail, a single block, strided blocks, diagonal only, query-head
    # groups, odd unions.
    (1, 192, 2, 2, 64, lg.Pattern(64, 1, 1, 0)),
    (1, 64, 1, 1, 64, lg.Pattern(64, 1, 1, 0)),
    (1, 2048, 2, 2, 64, lg.Pattern(64, 1, 16, 4)),
    (1, 1280, 2, 2, 64, lg.Pattern(64, 0, 1, 0)),
    (1, 640, 2, 1, 64, lg.Pattern(64, 2, 3, 0)),
    (2, 896, 4, 4, 64, lg.Pattern(64, 0, 3, 0)),
]


@pytest.mark.parametrize("B,S,H,Hkv,D,pat", SMALL)
def test_fwd_matches_oracle_small(B, S, H, Hkv, D, pat):
    q, k, v = si.prefill_inputs(B, S, H, Hkv, D)
    scale = 1.0 / math.sqrt(D)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = run_fwd(pat, qd, kd, vd, scale)
    ro, rlse = oracle.attention_forward(q, k, v, oracle.Pattern(*pat), scale)
    assert_close("O", o.float().cpu().numpy(), ro)
    assert_lse("LSE", lse.cpu().numpy(), rlse)
    # fp32 output: the same accumulators without the bf16 rounding.
    o32, lse32 = run_fwd(pat, qd, kd, vd, scale, torch.float32)
    assert_close("O fp32", o32.cpu().numpy(), ro)
    assert torch.equal(lse32, lse)
    assert torch.equal(o32.to(torch.bfloat16), o)


@pytest.mark.parametrize("D", [64, 128])
def test_fwd_lazy_rescale_with_growing_scores(D):
    """Keys whose scale grows along the sequence push each row's running max up
    by more than 2^8 from one KV chunk to the next, so O is rescaled at nearly
    every chunk, at both head dims. Such rows are carried by
    a few keys, so the bf16 rounding of their P (2^-9 relative) no longer
    averages out; V is scaled by 1/4 to keep that rounding well inside the
    bound -- the growth of the scores, set by K alone, is unchanged."""
    B, S, H = 1, 1024, 2
    q, k, v = si.prefill_inputs(B, S, H, H, D)
    k = (k.float() * torch.linspace(1.0, 60.0, S).view(1, S, 1, 1)).to(torch.bfloat16)
    v = (v.float() * 0.25).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_fwd(lg.Pattern.full(64), q.cuda(), k.cuda(), v.cuda(), scale, torch.float32)
    ro, rlse = oracle.attention_forward(q, k, v, oracle.Pattern(*lg.Pattern.full(64)), scale)
    assert_close("O fp32", o.cpu().numpy(), ro)
    assert_lse("LSE", lse.cpu().numpy(), rlse)


def test_fwd_repeatable():
    q, k, v = si.prefill_inputs(1, 512, 2, 2, 128)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = run_fwd(lg.Pattern(64, 1, 3, 0), qd, kd, vd, 0.088)
    o2, l2 = run_fwd(lg.Pattern(64, 1, 3, 0), qd, kd, vd, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def sampled_blocks(nqb, seed=5):
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(2, nqb - 2), size=8, replace=False)
    return sorted({0, 1, nqb - 2, nqb - 1, *mid.tolist()})


LARGE = [
    ("32K sink+window", 32768, lg.Pattern(64, 1, 64, 0)),
    ("32K dense", 32768, lg.Pattern.full(64)),
    ("128K block-sparse", 131072, lg.Pattern(64, 1, 16, 32)),
]


@pytest.mark.parametrize("name,S,pat", LARGE)
def test_fwd_full_size_sampled(name, S, pat):
    B, H, D = 1, 32, 128
    dev = torch.device("cuda")
    q, k, v = si.prefill_inputs_device(B, S, H, H, D, dev)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_fwd(pat, q, k, v, scale)
    rows = np.concatenate([np.arange(b * 64, (b + 1) * 64) for b in sampled_blocks(S // 64)])
    op = oracle.Pattern(*pat)
    for h in (0, H - 1):
        qh, kh, vh = (t[0, :, h].float().cpu().numpy() for t in (q, k, v))
        ro, rl = oracle.attention_rows(qh, kh, vh, rows, op, scale)
        assert_close(f"{name} O h{h}", o[0, rows, h].float().cpu().numpy(), ro)
        assert_lse(f"{name} LSE h{h}", lse[0, h, rows].cpu().numpy(), rl)


def run_fwd_pair(pattern, q, k, v, scale, o_dtype=torch.bfloat16):
    B, S, H, D = q.shape
    o = torch.empty(q.shape, dtype=o_dtype, device=q.device)
    lse = torch.empty(B, H, S, dtype=torch.float32, device=q.device)
    lg.lg_sparse_attn_fwd_pair(pattern, q, k, v, o, lse, scale)
    torch.cuda.synchronize()
    assert lg.lg_device_status(q.device.index or 0) == 0
    return o, lse


@pytest.mark.parametrize("B,S,H,Hkv,D,pat", [c for c in SMALL if c[4] == 128])
def test_fwd_pair_matches_oracle_small(B, S, H, Hkv, D, pat):
    q, k, v = si.prefill_inputs(B, S, H, Hkv, D)
    scale = 1.0 / math.sqrt(D)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o32, lse = run_fwd_pair(pat, qd, kd, vd, scale, torch.float32)
    ro, rlse = oracle.attention_forward(q, k, v, oracle.Pattern(*pat), scale)
    assert_close("O fp32", o32.cpu().numpy(), ro)
    assert_lse("LSE", lse.cpu().numpy(), rlse)
    o16, lse16 = run_fwd_pair(pat, qd, kd, vd, scale)
    assert torch.equal(lse16, lse)
    assert torch.equal(o32.to(torch.bfloat16), o16)
    # The single-CTA forward computes the same rows. A 512-row span pairs other KV blocks into
    # chunks than a 256-row span does, so the bf16 rounding of P and the lazy-rescale points
    # differ: the two outputs agree to the parity bound, not bit for bit.
    o1, l1 = run_fwd(pat, qd, kd, vd, scale, torch.float32)
    assert_close("O pair vs single", o32.cpu().numpy(), o1.cpu().numpy())
    assert float((l1 - lse).abs().max()) <= 1e-5


def test_fwd_pair_rejects_head_dim_64():
    q, k, v = si.prefill_inputs(1, 256, 2, 2, 64)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lg.LgError) as e:
        lg.lg_sparse_attn_fwd_pair(lg.Pattern(64, 1, 2, 0), q.cuda(), k.cuda(), v.cuda(), o, None, 0.125)
    assert e.value.status == 2


@pytest.mark.parametrize("name,S,pat", [LARGE[1], LARGE[2]])
def test_fwd_pair_full_size_sampled(name, S, pat):
    B, H, D = 1, 32, 128
    dev = torch.device("cuda")
    q, k, v = si.prefill_inputs_device(B, S, H, H, D, dev)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_fwd_pair(pat, q, k, v, scale)
    rows = np.concatenate([np.arange(b * 64, (b + 1) * 64) for b in sampled_blocks(S // 64)])
    op = oracle.Pattern(*pat)
    for h in (0, H - 1):
        qh, kh, vh = (t[0, :, h].float().cpu().numpy() for t in (q, k, v))
        ro, rl = oracle.attention_rows(qh, kh, vh, rows, op, scale)
        assert_close(f"{name} pair O h{h}", o[0, rows, h].float().cpu().numpy(), ro)
        assert_lse(f"{name} pair LSE h{h}", lse[0, h, rows].cpu().numpy(), rl)


def test_fwd_head_dim_64_full_size_sampled():
    """The head-dim-64 workload bench.py times: 32K sink+window, B1 H32 D64."""
    B, S, H, D = 1, 32768, 32, 64
    pat = lg.Pattern(64, 1, 64, 0)
    dev = torch.device("cuda")
    q, k, v = si.prefill_inputs_device(B, S, H, H, D, dev)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_fwd(pat, q, k, v, scale)
    rows = np.concatenate([np.arange(b * 64, (b + 1) * 64) for b in sampled_blocks(S // 64)])
    op = oracle.Pattern(*pat)
    for h in (0, H - 1):
        qh, kh, vh = (t[0, :, h].float().cpu().numpy() for t in (q, k, v))
        ro, rl = oracle.attention_rows(qh, kh, vh, rows, op, scale)
        assert_close(f"D64 O h{h}", o[0, rows, h].float().cpu().numpy(), ro)
        assert_lse(f"D64 LSE h{h}", lse[0, h, rows].cpu().numpy(), rl)
