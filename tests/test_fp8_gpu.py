"""Forward with Q and K in fp8 e4m3 (lg_sparse_attn_fwd_fp8qk) through the
C-ABI vs the fp64 oracle.

The kernel computes exact attention over the dequantised Q and K (q8 *
q_descale, k8 * k_descale), so the oracle is given exactly those values: the
comparison checks the kernel, not the quantisation. Quantisation uses scales
other than one so the descales are exercised. Small shapes are compared in
full; the 32K dense workload the bench times on sampled rows.
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

QS, KS = 4.0, 2.0  # quantisation scales: q8 = e4m3(q * QS), descale 1 / QS


def quantise(x, s):
    x8 = (x.float() * s).to(torch.float8_e4m3fn)
    return x8, x8.float() / s  # the fp8 tensor and the exact values it stands for


def run(pat, q8, k8, v, scale, odt):
    B, S, H, D = q8.shape
    o = torch.empty(B, S, H, D, dtype=odt, device="cuda")
    lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
    lg.lg_sparse_attn_fwd_fp8qk(pat, q8, k8, v, 1.0 / QS, 1.0 / KS, o, lse, scale)
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0
    return o, lse


CASES = [
    # B, S, H, Hkv, pattern, O dtype
    (1, 1024, 4, 4, (64, 1, 4, 0), torch.float32),
    (2, 640, 4, 2, (64, 0, 2**31 - 1, 0), torch.float32),
    (1, 2048, 2, 2, (64, 1, 16, 4), torch.float32),
    (1, 1024, 2, 1, (64, 1, 4, 0), torch.bfloat16),
    (1, 192, 2, 2, (64, 1, 1, 0), torch.float32),
]


@pytest.mark.parametrize("B,S,H,Hkv,pat,odt", CASES)
def test_fp8qk_forward_matches_oracle_on_dequantised_inputs(B, S, H, Hkv, pat, odt):
    D = 128
    q, k, v = si.prefill_inputs(B, S, H, Hkv, D, seed=si.SEED_BASE + 400)
    q8, qd = quantise(q, QS)
    k8, kd = quantise(k, KS)
    scale = 1.0 / math.sqrt(D)
    o, lse = run(pat, q8.cuda(), k8.cuda(), v.cuda(), scale, odt)
    ro, rl = oracle.attention_forward(qd, kd, v, oracle.Pattern(*pat), scale)
    assert_close("O", o.float().cpu().numpy(), ro)
    assert np.max(np.abs(lse.cpu().numpy() - rl)) <= LSE_TOL


def test_fp8qk_dense_32k_sampled():
    B, S, H, D = 1, 32768, 32, 128
    pat = (64, 0, 2**31 - 1, 0)
    dev = torch.device("cuda")
    q = si.device_normal((B, S, H, D), si.SEED_BASE + 0, dev)
    k = si.device_normal((B, S, H, D), si.SEED_BASE + 1, dev)
    v = si.device_normal((B, S, H, D), si.SEED_BASE + 2, dev)
    q8, qd = quantise(q, QS)
    k8, kd = quantise(k, KS)
    scale = 1.0 / math.sqrt(D)
    o, lse = run(pat, q8, k8, v, scale, torch.bfloat16)
    nqb = S // 64
    rows = np.concatenate([np.arange(i * 64, i * 64 + 64) for i in (0, 5, nqb // 2, nqb - 1)])
    op = oracle.Pattern(*pat)
    for h in (0, H - 1):
        qh, kh, vh = (t[0, :, h].cpu().numpy() for t in (qd, kd, v.float()))
        ro, rl = oracle.attention_rows(qh, kh, vh, rows, op, scale)
        assert_close(f"O h{h}", o[0, rows, h].float().cpu().numpy(), ro)
        assert np.max(np.abs(lse[0, h, rows].cpu().numpy() - rl)) <= LSE_TOL
