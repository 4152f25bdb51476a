"""Decode parity: the split-KV decode kernel through the C-ABI vs the fp64 oracle.

The fp32 output mode is compared with the oracle at the stated bound, and the
bf16 output is checked to be exactly its round-to-nearest-even. Covers ragged
cache lengths (1 .. Lmax), forced and automatic split counts,
GQA group sizes 1/2/4/8, D = 64 and 128, a zero-length cache, the full
batch-32 sparse-layer workload (compared in full) and the batch-32
131072-row full-layer workload (compared on sampled (b, h) rows).
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


def run_decode(q, kc, vc, lens, scale, num_splits=0):
    """Runs the decode twice, with an fp32 and with a bf16 output. Returns the
    fp32 output (compared with the unrounded oracle) after checking that the
    bf16 output is exactly its round-to-nearest-even and the LSEs agree."""
    B, H, D = q.shape
    Lmax, Hkv = kc.shape[1], kc.shape[2]
    nbytes = lg.lg_sparse_decode_workspace(B, H, Hkv, D, Lmax, num_splits)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    outs = []
    for dt in (torch.float32, torch.bfloat16):
        o = torch.empty(B, H, D, dtype=dt, device=q.device)
        lse = torch.empty(B, H, dtype=torch.float32, device=q.device)
        lg.lg_sparse_decode(q, kc, vc, lens, o, lse, scale, num_splits=num_splits, workspace=ws)
        outs.append((o, lse))
    torch.cuda.synchronize()
    assert lg.lg_device_status(q.device.index or 0) == 0
    (o32, lse), (o16, lse16) = outs
    assert torch.equal(o16.view(torch.int16), o32.to(torch.bfloat16).view(torch.int16))
    assert torch.equal(lse, lse16)
    return o32, lse


CASES = [
    # B, H, Hkv, D, Lmax, splits
    (3, 4, 2, 128, 1000, 0),
    (3, 4, 2, 128, 1000, 1),
    (3, 4, 2, 128, 1000, 7),
    (2, 8, 1, 128, 777, 0),
    (2, 8, 2, 64, 513, 3),
    (4, 16, 16, 64, 300, 0),
    (2, 4, 4, 128, 5000, 64),
]


@pytest.mark.parametrize("B,H,Hkv,D,Lmax,ns", CASES)
def test_decode_matches_oracle_ragged(B, H, Hkv, D, Lmax, ns):
    lens = si.ragged_lens(B, Lmax)
    lens[0] = 1
    q, kc, vc, cl = si.decode_inputs(B, H, Hkv, D, Lmax, lens=lens)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_decode(q.cuda(), kc.cuda(), vc.cuda(), cl.cuda(), scale, ns)
    ro, rl = oracle.decode(q, kc, vc, lens, scale)
    assert_close("o", o.cpu().numpy(), ro)
    assert_lse("lse", lse.cpu().numpy(), rl)


def test_decode_zero_length_is_empty():
    q, kc, vc, cl = si.decode_inputs(2, 2, 2, 128, 256, lens=[0, 256])
    o, lse = run_decode(q.cuda(), kc.cuda(), vc.cuda(), cl.cuda(), 0.1, 4)
    assert torch.all(o[0] == 0) and torch.all(torch.isinf(lse[0])) and torch.all(lse[0] < 0)
    ro, rl = oracle.decode(q[1:], kc[1:], vc[1:], [256], 0.1)
    assert_close("o", o[1:].cpu().numpy(), ro)


def test_decode_sparse_layer_full_size():
    B, H, D, L = 32, 32, 128, 4160  # 64 sink + 4096 window rows
    q, kc, vc, cl = si.decode_inputs(B, H, H, D, L)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_decode(q.cuda(), kc.cuda(), vc.cuda(), cl.cuda(), scale)
    ro, rl = oracle.decode(q, kc, vc, cl.numpy(), scale)
    assert_close("o", o.cpu().numpy(), ro)
    assert_lse("lse", lse.cpu().numpy(), rl)


def test_decode_full_layer_full_size_sampled():
    B, H, D, L = 32, 32, 128, 131072
    dev = torch.device("cuda")
    q, kc, vc, cl = si.decode_inputs_device(B, H, H, D, L, dev)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_decode(q, kc, vc, cl, scale)
    for b, h in ((0, 0), (5, 17), (31, 31), (16, 3)):
        ro, rl = oracle.decode(q[b:b + 1, h:h + 1].cpu(), kc[b:b + 1, :, h:h + 1].cpu(),
                               vc[b:b + 1, :, h:h + 1].cpu(), [L], scale)
        assert_close(f"o[{b},{h}]", o[b, h].cpu().numpy(), ro[0, 0])
        assert_lse(f"lse[{b},{h}]", lse[b, h].cpu().numpy(), rl[0, 0])


def test_gqa_decode_at_bench_size_sampled():
    """Grouped-query decode (H32, Hkv8: the tensor-core path) at the batch-32,
    4160-row size the bench times, ragged lengths: sampled (b, h) vs the oracle."""
    B, H, Hkv, D, L = 32, 32, 8, 128, 4160
    dev = torch.device("cuda")
    lens = [L - 61 * b for b in range(B)]
    q, kc, vc, cl = si.decode_inputs_device(B, H, Hkv, D, L, dev, lens=lens)
    scale = 1.0 / math.sqrt(D)
    o, lse = run_decode(q, kc, vc, cl, scale)
    G = H // Hkv
    for b, h in ((0, 0), (5, 17), (31, 31), (16, 3), (9, 12)):
        n = lens[b]
        ro, rl = oracle.decode(q[b:b + 1, h:h + 1].cpu(), kc[b:b + 1, :n, h // G:h // G + 1].cpu(),
                               vc[b:b + 1, :n, h // G:h // G + 1].cpu(), np.array([n]), scale)
        assert_close(f"o[{b},{h}]", o[b, h].cpu().numpy(), ro[0, 0])
        assert_lse(f"lse[{b},{h}]", lse[b, h].cpu().numpy(), rl[0, 0])
