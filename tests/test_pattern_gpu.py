"""The block iterator the kernels run, executed on the device, compared bit for
bit with the oracle's token-scan block lists (forward: per 64- or 128-row query
tile, the union of its blocks' KV lists plus per-block membership; backward:
per KV tile, the union of the query lists)."""

import numpy as np
import pytest
import torch

import oracle
import attention_sink_long_b200 as lg

pytestmark = pytest.mark.gpu

PATTERNS = [lg.Pattern(64, 1, 4, 0), lg.Pattern(64, 1, 16, 32), lg.Pattern(64, 0, 1, 0), lg.Pattern(64, 0, 2, 3),
            lg.Pattern(64, 3, 2, 5), lg.Pattern.full(64), lg.Pattern(64, 1, 64, 0), lg.Pattern(64, 40, 1, 0)]


def expected(p, S, tile_blocks, transpose):
    op = oracle.Pattern(*p)
    ptr, idx = (oracle.block_lists_t if transpose else oracle.block_lists)(S, op)
    nqb = S // 64
    tiles = []
    for lo in range(0, nqb, tile_blocks):
        members = {}
        for t in range(tile_blocks):
            if lo + t >= nqb:
                continue
            for j in idx[ptr[lo + t]:ptr[lo + t + 1]]:
                members[int(j)] = members.get(int(j), 0) | (1 << t)
        tiles.append([(j << 2) | m for j, m in sorted(members.items())])
    return tiles


@pytest.mark.parametrize("p", PATTERNS)
@pytest.mark.parametrize("S", [64, 192, 4096])
@pytest.mark.parametrize("tile_blocks", [1, 2])
@pytest.mark.parametrize("transpose", [0, 1])
def test_device_iterator_bit_exact(p, S, tile_blocks, transpose):
    cap = S // 64
    ntiles = (S // 64 + tile_blocks - 1) // tile_blocks
    out = torch.full((ntiles * (cap + 1),), -7, dtype=torch.int32, device="cuda")
    lg.lg_pattern_iterate_device(p, S, tile_blocks, transpose, out, cap)
    torch.cuda.synchronize()
    got = out.cpu().numpy().reshape(ntiles, cap + 1)
    exp = expected(p, S, tile_blocks, transpose)
    for u in range(ntiles):
        n = int(got[u, 0])
        assert n == len(exp[u]), (u, n, len(exp[u]))
        assert got[u, 1:1 + n].tolist() == exp[u]
