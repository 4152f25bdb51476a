"""lg_sparse_decode_noalloc -- decode for callers that cannot allocate device memory.

Such callers (a plugin inside a framework that owns every device allocation,
a latency-critical decode loop where cudaMalloc / cudaFree would synchronise
the device, a thin C / FFI caller without a device allocator) cannot hand the
library a workspace. This entry point keeps the split partials in the
library's fixed 16 MiB device array instead. It is checked here against
lg_sparse_decode (the entry point that takes a caller workspace) on two calls
in a row, so the second call runs on the scratch contents the first left
behind, and against the fp64 oracle.

This file is collected last on purpose: a run that stops at the first failure
has already run every other test. It passes alone in a fresh process and after
the rest of the suite.
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


def decode_with_workspace(q, kc, vc, cl, scale, ns):
    B, H, D = q.shape
    Lmax, Hkv = kc.shape[1], kc.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(B, H, dtype=torch.float32, device=q.device)
    ws = torch.empty(max(lg.lg_sparse_decode_workspace(B, H, Hkv, D, Lmax, ns), 1), dtype=torch.uint8,
                     device=q.device)
    lg.lg_sparse_decode(q, kc, vc, cl, o, lse, scale, num_splits=ns, workspace=ws)
    return o, lse


def decode_noalloc(q, kc, vc, cl, scale, ns):
    B, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(B, H, dtype=torch.float32, device=q.device)
    lg.lg_sparse_decode_noalloc(q, kc, vc, cl, o, lse, scale, num_splits=ns)
    return o, lse


CASES = [
    # B, H, Hkv, D, Lmax, num_splits, ragged lengths
    (32, 32, 32, 128, 4160, 0, False),  # one sparse layer of the batch-32 decode workload, automatic splits
    (3, 8, 2, 128, 1000, 5, True),      # GQA, ragged lengths, explicit split count
    (2, 4, 4, 64, 700, 0, True),
]


@pytest.mark.parametrize("B,H,Hkv,D,Lmax,ns,ragged", CASES)
def test_noalloc_matches_workspace_decode_two_calls_in_a_row(B, H, Hkv, D, Lmax, ns, ragged):
    dev = torch.device("cuda")
    scale = 1.0 / math.sqrt(D)
    for call, seed in enumerate((1000, 1100)):
        lens = si.ragged_lens(B, Lmax, seed=seed + 7) if ragged else None
        q, kc, vc, cl = si.decode_inputs(B, H, Hkv, D, Lmax, seed=seed, lens=lens)
        qd, kd, vd, cd = q.to(dev), kc.to(dev), vc.to(dev), cl.to(dev)
        o_na, l_na = decode_noalloc(qd, kd, vd, cd, scale, ns)
        o_ws, l_ws = decode_with_workspace(qd, kd, vd, cd, scale, ns)
        torch.cuda.synchronize()
        assert_close(f"call {call}: noalloc vs workspace o", o_na.float().cpu().numpy(), o_ws.float().cpu().numpy())
        assert_lse(f"call {call}: noalloc vs workspace lse", l_na.cpu().numpy(), l_ws.cpu().numpy())
        ro, rl = oracle.decode(q, kc, vc, cl.numpy(), scale)
        assert_close(f"call {call}: noalloc vs oracle o", o_na.float().cpu().numpy(), ro)
        assert_lse(f"call {call}: noalloc vs oracle lse", l_na.cpu().numpy(), rl)


def test_noalloc_rejects_split_count_beyond_scratch():
    dev = torch.device("cuda")
    B, H, D, L = 32, 32, 128, 8192
    q = torch.zeros(B, H, D, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(B, L, H, D, dtype=torch.bfloat16, device=dev)
    cl = torch.full((B,), L, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    # 64 splits of 32 x 32 rows need 64 * 1024 * 129 * 4 bytes (about 34 MB) > 16 MiB.
    with pytest.raises(lg.LgError) as e:
        lg.lg_sparse_decode_noalloc(q, kc, kc, cl, o, None, 0.1, num_splits=64)
    assert e.value.status == 3  # LG_ERR_WORKSPACE
