"""The block iterators the kernels run, executed on the device, compared bit for
bit with the oracle's token-scan block lists:

* forward unions (mode 0): per tile of 1, 2, 4 or 8 query blocks, the union of
  their KV lists with per-block membership;
* backward unions (mode 1): per tile of 1 or 2 KV blocks, the union of their
  query lists;
* the forward kernels' chunked walk (mode 2): the union list of a 4- or
  8-block query span, in order, cut into chunks of two consecutive listed
  blocks (the last chunk holds one block when the list is odd);
* the backward kernels' KV tiles (mode 3): every KV block in exactly one tile;
  blocks that every later query sees (sink and strided blocks, found with the
  oracle's token predicate) paired first, ascending, then the window-only
  blocks, ascending; each tile walks exactly the query blocks of the union of
  its two blocks' transposed lists, with per-block membership.
"""

import functools

import numpy as np
import pytest
import torch

import oracle
import attention_sink_long_b200 as lg

pytestmark = pytest.mark.gpu

PATTERNS = [lg.Pattern(64, 1, 4, 0), lg.Pattern(64, 1, 16, 32), lg.Pattern(64, 0, 1, 0), lg.Pattern(64, 0, 2, 3),
            lg.Pattern(64, 3, 2, 5), lg.Pattern.full(64), lg.Pattern(64, 1, 64, 0), lg.Pattern(64, 40, 1, 0)]
SIZES = [64, 192, 4096]
# The workload sizes: the 32K sink+window / dense patterns and the 128K block-sparse pattern.
LARGE = [(lg.Pattern(64, 1, 64, 0), 32768), (lg.Pattern.full(64), 32768), (lg.Pattern(64, 1, 16, 32), 131072)]


@functools.lru_cache(maxsize=None)
def lists(p, S, transpose):
    """The oracle's CSR (transpose=0) or CSC (transpose=1) block lists, as a list of lists."""
    ptr, idx = (oracle.block_lists_t if transpose else oracle.block_lists)(S, oracle.Pattern(*p))
    return [idx[ptr[i]:ptr[i + 1]].tolist() for i in range(len(ptr) - 1)]


def union_with_membership(L, lo, n):
    members = {}
    for t in range(n):
        if lo + t >= len(L):
            continue
        for j in L[lo + t]:
            members[j] = members.get(j, 0) | (1 << t)
    return sorted(members.items())


def run(p, S, tile_blocks, mode, cap, ntiles):
    out = torch.full((ntiles * (cap + 1),), -7, dtype=torch.int32, device="cuda")
    lg.lg_pattern_iterate_device(p, S, tile_blocks, mode, out, cap)
    torch.cuda.synchronize()
    return out.cpu().numpy().reshape(ntiles, cap + 1)


def check_union(p, S, tile_blocks, transpose):
    nqb = S // 64
    cap = nqb
    ntiles = (nqb + tile_blocks - 1) // tile_blocks
    got = run(p, S, tile_blocks, transpose, cap, ntiles)
    L = lists(p, S, transpose)
    for u in range(ntiles):
        exp = [(j << 8) | m for j, m in union_with_membership(L, u * tile_blocks, tile_blocks)]
        n = int(got[u, 0])
        assert n == len(exp), (u, n, len(exp))
        assert got[u, 1:1 + n].tolist() == exp, u


def check_chunks(p, S, span):
    nqb = S // 64
    cap = 2 * nqb
    ntiles = (nqb + span - 1) // span
    got = run(p, S, span, 2, cap, ntiles)
    L = lists(p, S, 0)
    for u in range(ntiles):
        un = [(j << 8) | m for j, m in union_with_membership(L, u * span, span)]
        exp = []
        for c in range(0, len(un), 2):
            exp += [un[c], un[c + 1] if c + 1 < len(un) else -1]
        n = int(got[u, 0])
        assert n == len(exp), (u, n, len(exp))
        assert got[u, 1:1 + n].tolist() == exp, u


def check_pairing(p, S):
    nqb = S // 64
    op = oracle.Pattern(*p)
    LT = [set(x) for x in lists(p, S, 1)]
    # A block every later query sees: the first query block past its window still attends to it.
    kb = np.arange(nqb, dtype=np.int64)
    is_glob = oracle.allowed((kb + min(op.local_blocks, 2**30)) * 64, kb * 64, op)
    seq = kb[is_glob].tolist() + kb[~is_glob].tolist()
    ntiles = (nqb + 1) // 2
    cap = nqb + 4
    got = run(p, S, 2, 3, cap, ntiles)
    for u in range(ntiles):
        kx = seq[2 * u]
        ky = seq[2 * u + 1] if 2 * u + 1 < nqb else -1
        qs = LT[kx] | (LT[ky] if ky >= 0 else set())
        q_first, last = min(qs), max(qs)
        exp = [kx, ky, q_first, last]
        for i in range(q_first, last + 1):
            exp.append((i << 8) | (1 if i in LT[kx] else 0) | (2 if ky >= 0 and i in LT[ky] else 0))
        n = int(got[u, 0])
        assert n == len(exp), (u, n, len(exp))
        assert got[u, 1:1 + n].tolist() == exp, u


@pytest.mark.parametrize("p", PATTERNS)
@pytest.mark.parametrize("S", SIZES)
@pytest.mark.parametrize("tile_blocks", [1, 2, 4, 8])
def test_forward_union_bit_exact(p, S, tile_blocks):
    check_union(p, S, tile_blocks, 0)


@pytest.mark.parametrize("p", PATTERNS)
@pytest.mark.parametrize("S", SIZES)
@pytest.mark.parametrize("tile_blocks", [1, 2])
def test_backward_union_bit_exact(p, S, tile_blocks):
    check_union(p, S, tile_blocks, 1)


@pytest.mark.parametrize("p", PATTERNS)
@pytest.mark.parametrize("S", SIZES)
@pytest.mark.parametrize("span", [4, 8])
def test_forward_chunk_walk_bit_exact(p, S, span):
    check_chunks(p, S, span)


@pytest.mark.parametrize("p", PATTERNS)
@pytest.mark.parametrize("S", SIZES)
def test_backward_tile_pairing_bit_exact(p, S):
    check_pairing(p, S)


@pytest.mark.parametrize("p,S", LARGE, ids=["sink_window_32k", "dense_32k", "block_sparse_128k"])
def test_iterators_at_workload_sizes(p, S):
    check_union(p, S, 4, 0)
    check_union(p, S, 2, 1)
    check_chunks(p, S, 4)
    check_chunks(p, S, 8)
    check_pairing(p, S)
