"""lg_sparse_decode_noalloc -- decode for callers that cannot allocate device memory.

Such callers (a plugin inside a framework that owns every device allocation,
a latency-critical decode loop where cudaMalloc / cudaFree would synchronise
the device, a thin C / FFI caller without a device allocator) cannot hand the
library a workspace. This entry point keeps the split partials in the
library's fixed 16 MiB device array instead. It runs the same kernel with the
same split count as lg_sparse_decode (the entry point that takes a caller
workspace), so the two outputs must be identical bit for bit; that is checked
on two calls in a row, so the second call runs on the scratch contents the
first left behind. The output is also checked against the fp64 oracle.

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

SCRATCH = 16 << 20  # LG_DECODE_NOALLOC_SCRATCH_BYTES


def decode_with_workspace(q, kc, vc, cl, scale, ns, dtype):
    B, H, D = q.shape
    Lmax, Hkv = kc.shape[1], kc.shape[2]
    o = torch.empty(B, H, D, dtype=dtype, device=q.device)
    lse = torch.empty(B, H, dtype=torch.float32, device=q.device)
    ws = torch.empty(max(lg.lg_sparse_decode_workspace(B, H, Hkv, D, Lmax, ns), 1), dtype=torch.uint8,
                     device=q.device)
    lg.lg_sparse_decode(q, kc, vc, cl, o, lse, scale, num_splits=ns, workspace=ws)
    return o, lse


def decode_noalloc(q, kc, vc, cl, scale, ns, dtype):
    B, H, D = q.shape
    o = torch.empty(B, H, D, dtype=dtype, device=q.device)
    lse = torch.empty(B, H, dtype=torch.float32, device=q.device)
    lg.lg_sparse_decode_noalloc(q, kc, vc, cl, o, lse, scale, num_splits=ns)
    return o, lse


def noalloc_splits(B, H, Hkv, D, L):
    """The split count the no-allocation entry point uses with num_splits == 0:
    the automatic count, lowered until the partials fit the fixed array."""
    ns = lg.lg_sparse_decode_splits(B, H, Hkv, D, L)
    while ns > 1 and lg.lg_sparse_decode_workspace(B, H, Hkv, D, L, ns) > SCRATCH:
        ns -= 1
    return ns


CASES = [
    # B, H, Hkv, D, Lmax, num_splits, ragged lengths, output dtype
    (32, 32, 32, 128, 4160, 0, False, torch.bfloat16),  # one sparse layer of the batch-32 decode, automatic splits
    (3, 8, 2, 128, 1000, 5, True, torch.float32),       # GQA, ragged lengths, explicit split count, fp32 output
    (2, 4, 4, 64, 700, 0, True, torch.bfloat16),
]


@pytest.mark.parametrize("B,H,Hkv,D,Lmax,ns,ragged,dtype", CASES)
def test_noalloc_matches_workspace_decode_two_calls_in_a_row(B, H, Hkv, D, Lmax, ns, ragged, dtype):
    dev = torch.device("cuda")
    scale = 1.0 / math.sqrt(D)
    for call, seed in enumerate((1000, 1100)):
        lens = si.ragged_lens(B, Lmax, seed=seed + 7) if ragged else None
        q, kc, vc, cl = si.decode_inputs(B, H, Hkv, D, Lmax, seed=seed, lens=lens)
        qd, kd, vd, cd = q.to(dev), kc.to(dev), vc.to(dev), cl.to(dev)
        o_na, l_na = decode_noalloc(qd, kd, vd, cd, scale, ns, dtype)
        o_ws, l_ws = decode_with_workspace(qd, kd, vd, cd, scale, ns, dtype)
        torch.cuda.synchronize()
        assert torch.equal(o_na, o_ws), f"call {call}: o differs from the workspace decode"
        assert torch.equal(l_na, l_ws), f"call {call}: lse differs from the workspace decode"
        ro, rl = oracle.decode(q, kc, vc, cl.numpy(), scale)
        assert_close(f"call {call}: noalloc vs oracle o", o_na.float().cpu().numpy(), ro)
        assert_lse(f"call {call}: noalloc vs oracle lse", l_na.cpu().numpy(), rl)


def test_noalloc_lowers_the_automatic_split_count_to_fit():
    """A cache whose automatic split count needs more than 16 MiB of partials:
    160 sequences of 32768 rows, 8 query heads on one KV head (2.7 GB of K/V;
    32 pieces, about 21 MB). The entry point lowers the count until the partials
    fit and must equal lg_sparse_decode run with that lowered count."""
    B, H, Hkv, D, L = 160, 8, 1, 128, 32768
    auto = lg.lg_sparse_decode_splits(B, H, Hkv, D, L)
    assert lg.lg_sparse_decode_workspace(B, H, Hkv, D, L, auto) > SCRATCH
    ns = noalloc_splits(B, H, Hkv, D, L)
    assert 1 < ns < auto
    dev = torch.device("cuda")
    lens = [L - 97 * b for b in range(B)]
    q, kc, vc, cl = si.decode_inputs_device(B, H, Hkv, D, L, dev, lens=lens)
    scale = 1.0 / math.sqrt(D)
    for call in range(2):
        o_na, l_na = decode_noalloc(q, kc, vc, cl, scale, 0, torch.float32)
        o_ws, l_ws = decode_with_workspace(q, kc, vc, cl, scale, ns, torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(o_na, o_ws), call
        assert torch.equal(l_na, l_ws), call
    for b, h in ((0, 0), (77, 5), (159, 7)):
        n = lens[b]
        ro, rl = oracle.decode(q[b:b + 1, h:h + 1].cpu(), kc[b:b + 1, :n].cpu(), vc[b:b + 1, :n].cpu(),
                               np.array([n]), scale)
        assert_close(f"o[{b},{h}]", o_na[b, h].cpu().numpy(), ro[0, 0])
        assert_lse(f"lse[{b},{h}]", l_na[b, h].cpu().numpy(), rl[0, 0])


def test_noalloc_rejects_split_count_beyond_scratch():
    dev = torch.device("cuda")
    B, H, Hkv, D, L = 32, 32, 4, 128, 8192
    q = torch.zeros(B, H, D, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(B, L, Hkv, D, dtype=torch.bfloat16, device=dev)
    cl = torch.full((B,), L, dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    # 64 splits of 32 x 32 query rows need 64 * 1024 * 129 * 4 bytes (about 34 MB) > 16 MiB.
    with pytest.raises(lg.LgError) as e:
        lg.lg_sparse_decode_noalloc(q, kc, kc, cl, o, None, 0.1, num_splits=64)
    assert e.value.status == 3  # LG_ERR_WORKSPACE
