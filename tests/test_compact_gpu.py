"""Prefill -> decode hand-off parity: lg_kv_compact through the C-ABI vs the
fp64 oracle's reduced-cache rows (oracle.reduced_cache_rows).

The kernel copies values, so the check is bit-exact: every written cache row
equals the prompt row the oracle lists for that position, rows past the cache
length keep their previous contents, and cache_lens equals the oracle's row
count. The hand-off identity -- decoding token S over the reduced cache plus
its own K/V row equals prefill attention row S -- is checked through the
library's decode against the oracle's prefill row, at the decode tolerances.
Small shapes are compared in full; the 32K batch-32 hand-off on sampled batch
rows.
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

SENTINEL = -12345  # int16 bit pattern left in rows the call must not touch

CASES = [
    # B, S, Hkv, D, pattern
    (2, 4096, 4, 128, (64, 1, 64, 0)),        # window covers the whole prompt: every row kept
    (2, 8192, 4, 128, (64, 1, 16, 32)),       # block-sparse: sink, strided blocks, window
    (3, 1024, 2, 64, (64, 1, 4, 0)),          # the 1K attention-sink pattern, head dim 64
    (1, 2048, 1, 128, (64, 4, 8, 0)),         # several sink blocks
    (2, 4096, 8, 64, (64, 0, 1, 0)),          # no earlier block is visible: length 0
    (1, 64, 2, 128, (64, 1, 64, 0)),          # a one-block prompt
    (1, 4096, 2, 128, (64, 0, 2**31 - 1, 0)), # full layer: the whole prompt
    (2, 8192, 2, 128, (64, 0, 2, 3)),         # strided without sink, short window
]


def run_compact(pattern, k, v, extra_rows=64):
    B, S, Hkv, D = k.shape
    n = lg.lg_kv_compact_rows(pattern, S)
    Lmax = n + extra_rows
    kc = torch.full((B, Lmax, Hkv, D), SENTINEL, dtype=torch.int16, device=k.device).view(torch.bfloat16)
    vc = torch.full((B, Lmax, Hkv, D), SENTINEL, dtype=torch.int16, device=k.device).view(torch.bfloat16)
    lens = torch.full((B,), -1, dtype=torch.int32, device=k.device)
    lg.lg_kv_compact(pattern, k, v, kc, vc, lens)
    torch.cuda.synchronize()
    assert lg.lg_device_status(k.device.index or 0) == 0
    return n, kc, vc, lens


@pytest.mark.parametrize("B,S,Hkv,D,pat", CASES)
def test_compact_matches_oracle_rows(B, S, Hkv, D, pat):
    _, k, v = si.prefill_inputs(B, S, Hkv, Hkv, D)
    rows = oracle.reduced_cache_rows(S, oracle.Pattern(*pat))
    kd, vd = k.cuda(), v.cuda()
    n, kc, vc, lens = run_compact(pat, kd, vd)
    assert n == len(rows)
    assert torch.all(lens.cpu() == n)
    idx = torch.from_numpy(rows)
    assert torch.equal(kc[:, :n].cpu().view(torch.int16), k[:, idx].view(torch.int16))
    assert torch.equal(vc[:, :n].cpu().view(torch.int16), v[:, idx].view(torch.int16))
    assert torch.all(kc[:, n:].view(torch.int16) == SENTINEL)
    assert torch.all(vc[:, n:].view(torch.int16) == SENTINEL)


@pytest.mark.parametrize("pat,H,Hkv", [((64, 1, 4, 0), 4, 2), ((64, 1, 2, 4), 4, 4), ((64, 2, 3, 0), 8, 1)])
def test_handoff_then_decode_equals_prefill_row(pat, H, Hkv):
    B, S, D = 2, 1024, 128
    scale = 1.0 / math.sqrt(D)
    q, k, v = si.prefill_inputs(B, S + 64, H, Hkv, D)  # token S is the first decode token
    kd, vd = k[:, :S].contiguous().cuda(), v[:, :S].contiguous().cuda()
    n, kc, vc, lens = run_compact(pat, kd, vd)
    kc[:, n] = k[:, S].cuda()  # the decode token's own row, appended by the caller
    vc[:, n] = v[:, S].cuda()
    lens += 1
    o = torch.empty(B, H, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(lg.lg_sparse_decode_workspace(B, H, Hkv, D, kc.shape[1]), 1), dtype=torch.uint8,
                     device="cuda")
    lg.lg_sparse_decode(q[:, S].contiguous().cuda(), kc, vc, lens, o, lse, scale, workspace=ws)
    torch.cuda.synchronize()
    p = oracle.Pattern(*pat)
    g = H // Hkv
    for b in range(B):
        for h in range(H):
            qh, kh, vh = (t[b, :, hh].float().numpy() for t, hh in ((q, h), (k, h // g), (v, h // g)))
            ro, rl = oracle.attention_rows(qh, kh, vh, [S], p, scale)
            assert_close(f"o b{b} h{h}", o[b, h].float().cpu().numpy()[None], ro)
            assert abs(lse[b, h].item() - rl[0]) <= LSE_TOL


def test_compact_32k_batch32_sampled():
    B, S, Hkv, D = 32, 32768, 32, 128
    pat = (64, 1, 64, 0)
    dev = torch.device("cuda")
    k = si.device_normal((B, S, Hkv, D), si.SEED_BASE + 1, dev)
    v = si.device_normal((B, S, Hkv, D), si.SEED_BASE + 2, dev)
    rows = oracle.reduced_cache_rows(S, oracle.Pattern(*pat))
    n, kc, vc, lens = run_compact(pat, k, v)
    assert n == len(rows) == 4096
    assert torch.all(lens == n)
    idx = torch.from_numpy(rows).to(dev)
    for b in (0, 1, 17, 31):
        assert torch.equal(kc[b, :n].view(torch.int16), k[b, idx].view(torch.int16))
        assert torch.equal(vc[b, :n].view(torch.int16), v[b, idx].view(torch.int16))
    assert torch.all(kc[:, n:].view(torch.int16) == SENTINEL)
