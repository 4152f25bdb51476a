"""Paged decode cache through the C-ABI vs the fp64 oracle: the hand-off into
pages (lg_kv_compact_paged), the per-token append with ring reuse of the
window's pages (lg_kv_append_paged) and decode through the block table
(lg_sparse_decode_paged).

After the hand-off and after every appended token t, the cache read through
its block table (entries [0, ceil(len / 64)), the first cache_lens rows) must
equal, bit for bit and in order, the oracle's reduced-cache rows for position
t followed by row t itself: exactly the keys prefill attention row t may
attend. The paged decode of query t must match the oracle's prefill row t.
Pages come from a shuffled pool shared by the batch, and the sink+window case
runs hundreds of tokens past its prompt with only sink + local pages, so the
window's pages are reused as a ring. At the batch-32, 4160-row decode size the
paged decode equals the contiguous decode bit for bit (same rows in the same
order, same splits). States that break the rules are reported through
lg_device_status (bit 6) and left unchanged.
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
PAGED_BIT = 64


class Paged:
    """Device state of a paged cache with a shuffled page pool."""

    def __init__(self, B, MB, Hkv, D, spare_pages=7, seed=0):
        P = B * MB + spare_pages
        perm = torch.randperm(P, generator=torch.Generator().manual_seed(seed))[: B * MB]
        self.table = perm.view(B, MB).to(torch.int32).cuda()
        self.k_pool = torch.full((P, 64, Hkv, D), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        self.v_pool = torch.full((P, 64, Hkv, D), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        self.ids = torch.full((B, MB), -1, dtype=torch.int32, device="cuda")
        self.lens = torch.zeros(B, dtype=torch.int32, device="cuda")
        self.pos = torch.zeros(B, dtype=torch.int32, device="cuda")

    def state(self):
        return self.k_pool, self.v_pool, self.table, self.ids, self.lens, self.pos

    def gather(self, b):
        """The cache rows of sequence b in table order: (k, v) [n, Hkv, D] on the host."""
        n = int(self.lens[b])
        nb = (n + 63) // 64
        pages = self.table[b, :nb].long()
        k = self.k_pool[pages].reshape(nb * 64, *self.k_pool.shape[2:])[:n]
        v = self.v_pool[pages].reshape(nb * 64, *self.v_pool.shape[2:])[:n]
        return k.cpu(), v.cpu()


def expected_rows(t, p):
    """Keys prefill row t attends: the reduced cache of position t, then row t."""
    return np.concatenate([oracle.reduced_cache_rows(t, p), np.array([t], dtype=np.int64)])


def decode_paged(pc, q, scale, dtype=torch.bfloat16):
    B, H, D = q.shape
    Hkv = pc.k_pool.shape[2]
    MB = pc.table.shape[1]
    o = torch.empty(B, H, D, dtype=dtype, device="cuda")
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(lg.lg_sparse_decode_workspace(B, H, Hkv, D, 64 * MB), 1), dtype=torch.uint8, device="cuda")
    lg.lg_sparse_decode_paged(q, pc.k_pool, pc.v_pool, pc.table, pc.lens, o, lse, scale, workspace=ws)
    return o, lse


def check_decode_row(o32, o16, lse, q, k, v, t, p, scale, H, Hkv):
    """The fp32 output against the unrounded oracle at the stated bound; the bf16
    output must be exactly that fp32 output rounded to nearest even (the same
    kernel, the same splits, only the final store differs)."""
    assert torch.equal(o16.view(torch.int16), o32.to(torch.bfloat16).view(torch.int16)), t
    g = H // Hkv
    for b in range(q.shape[0]):
        for h in range(H):
            qh, kh, vh = (x[b, :, hh].float().numpy() for x, hh in ((q, h), (k, h // g), (v, h // g)))
            ro, rl = oracle.attention_rows(qh, kh[: t + 1], vh[: t + 1], [t], p, scale)
            assert_close(f"o t{t} b{b} h{h}", o32[b, h].cpu().numpy()[None], ro)
            assert abs(lse[b, h].item() - rl[0]) <= LSE_TOL, (t, b, h, lse[b, h].item(), rl[0])


RUNS = [
    # B, S (prompt), steps, H, Hkv, D, pattern, table entries
    (2, 512, 300, 4, 2, 128, (64, 1, 4, 0), 5),           # sink + window: 5 pages forever (a ring)
    (2, 1024, 200, 2, 2, 128, (64, 1, 2, 3), 12),         # strided blocks: the cache grows every 3 blocks
    (1, 256, 100, 4, 4, 64, (64, 0, 2**31 - 1, 0), 7),    # full layer: every block kept
    (2, 0, 200, 2, 1, 64, (64, 2, 2, 0), 4),              # no prompt: decoding from an empty cache
]


@pytest.mark.parametrize("B,S,steps,H,Hkv,D,pat,MB", RUNS)
def test_paged_decode_loop_matches_oracle(B, S, steps, H, Hkv, D, pat, MB):
    scale = 1.0 / math.sqrt(D)
    p = oracle.Pattern(*pat)
    q, k, v = si.prefill_inputs(B, S + steps, H, Hkv, D, seed=si.SEED_BASE + 300)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    pc = Paged(B, MB, Hkv, D)
    if S > 0:
        lg.lg_kv_compact_paged(pat, kd[:, :S].contiguous(), vd[:, :S].contiguous(), *pc.state())
        torch.cuda.synchronize()
        assert torch.all(pc.pos.cpu() == S)
        assert torch.all(pc.lens.cpu() == len(oracle.reduced_cache_rows(S, p)))
    for t in range(S, S + steps):
        lg.lg_kv_append_paged(pat, kd[:, t].contiguous(), vd[:, t].contiguous(), *pc.state())
        torch.cuda.synchronize()
        rows = torch.from_numpy(expected_rows(t, p))
        assert torch.all(pc.pos.cpu() == t + 1)
        assert torch.all(pc.lens.cpu() == len(rows)), (t, pc.lens.cpu(), len(rows))
        for b in range(B):
            gk, gv = pc.gather(b)
            assert torch.equal(gk.view(torch.int16), k[b, rows].view(torch.int16)), (t, b)
            assert torch.equal(gv.view(torch.int16), v[b, rows].view(torch.int16)), (t, b)
        # The decode of token t, at every block boundary and a sample between.
        if t % 64 in (0, 1, 63) or t % 29 == 0:
            o32, lse = decode_paged(pc, qd[:, t].contiguous(), scale, torch.float32)
            o16, lse16 = decode_paged(pc, qd[:, t].contiguous(), scale)
            torch.cuda.synchronize()
            assert torch.equal(lse, lse16)
            check_decode_row(o32, o16, lse, q, k, v, t, p, scale, H, Hkv)
    assert lg.lg_device_status(0) == 0


def test_sink_window_ring_never_needs_more_pages():
    """Sink + window over 40 blocks of decoding: sink_blocks + local_blocks table entries suffice."""
    B, H, Hkv, D = 1, 2, 2, 64
    pat = (64, 1, 3, 0)
    p = oracle.Pattern(*pat)
    steps = 40 * 64
    _, k, v = si.prefill_inputs(B, steps, H, Hkv, D, seed=si.SEED_BASE + 301)
    kd, vd = k.cuda(), v.cuda()
    pc = Paged(B, 4, Hkv, D, spare_pages=0)
    for t in range(steps):
        lg.lg_kv_append_paged(pat, kd[:, t].contiguous(), vd[:, t].contiguous(), *pc.state())
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0
    rows = torch.from_numpy(expected_rows(steps - 1, p))
    gk, gv = pc.gather(0)
    assert torch.equal(gk.view(torch.int16), k[0, rows].view(torch.int16))
    assert torch.equal(gv.view(torch.int16), v[0, rows].view(torch.int16))
    assert sorted(pc.table[0].tolist()) == list(range(4))  # the same four pages, permuted


@pytest.mark.parametrize("H,Hkv", [(32, 32), (32, 8)], ids=["mha", "gqa4"])
def test_paged_decode_equals_contiguous_bitwise_at_decode_size(H, Hkv):
    B, D, L = 32, 128, 4160
    MB = L // 64
    dev = torch.device("cuda")
    q = si.device_normal((B, H, D), si.SEED_BASE + 0, dev)
    kc = si.device_normal((B, L, Hkv, D), si.SEED_BASE + 1, dev)
    vc = si.device_normal((B, L, Hkv, D), si.SEED_BASE + 2, dev)
    lens = torch.tensor([L - 37 * b for b in range(B)], dtype=torch.int32, device=dev)
    P = B * MB + 3
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(5))[: B * MB].view(B, MB)
    table = perm.to(torch.int32).to(dev)
    k_pool = torch.empty(P, 64, Hkv, D, dtype=torch.bfloat16, device=dev)
    v_pool = torch.empty_like(k_pool)
    k_pool[perm.reshape(-1).to(dev)] = kc.view(B * MB, 64, Hkv, D)
    v_pool[perm.reshape(-1).to(dev)] = vc.view(B * MB, 64, Hkv, D)
    ws = torch.empty(lg.lg_sparse_decode_workspace(B, H, Hkv, D, L), dtype=torch.uint8, device=dev)
    o1 = torch.empty(B, H, D, dtype=torch.bfloat16, device=dev)
    l1 = torch.empty(B, H, dtype=torch.float32, device=dev)
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    lg.lg_sparse_decode(q, kc, vc, lens, o1, l1, 1 / math.sqrt(D), workspace=ws)
    lg.lg_sparse_decode_paged(q, k_pool, v_pool, table, lens, o2, l2, 1 / math.sqrt(D), workspace=ws)
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)
    # and one sampled (b, h) against the oracle
    G = H // Hkv
    for b, h in ((0, 0), (31, 17)):
        n = int(lens[b])
        kv = h // G
        ro, rl = oracle.decode(q[b:b + 1, h:h + 1].cpu(), kc[b:b + 1, :n, kv:kv + 1].cpu(),
                               vc[b:b + 1, :n, kv:kv + 1].cpu(), np.array([n]), 1 / math.sqrt(D))
        assert_close(f"o b{b} h{h}", o2[b, h].float().cpu().numpy()[None], ro[0])
        assert abs(l2[b, h].item() - rl[0, 0]) <= LSE_TOL


def test_page_outside_the_pool_is_reported_and_its_rows_left_out():
    B, H, Hkv, D = 1, 2, 2, 128
    scale = 1 / math.sqrt(D)
    q, k, v = si.prefill_inputs(B, 256, H, Hkv, D, seed=si.SEED_BASE + 302)
    pc = Paged(B, 4, Hkv, D, spare_pages=0)
    pc.table[0] = torch.tensor([2, 0, 3, 1], dtype=torch.int32)
    lg.lg_kv_compact_paged((64, 0, 2**31 - 1, 0), k.cuda(), v.cuda(), *pc.state())  # 4 blocks: 256 rows
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0
    pc.lens.fill_(256)
    pc.table[0, 2] = 4  # the pool has pages 0..3
    o, lse = decode_paged(pc, q[:, 200].contiguous().cuda(), scale, torch.float32)
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) & PAGED_BIT
    keep = np.r_[0:128, 192:256]
    ro, rl = oracle.decode(q[:, 200], k[:, keep], v[:, keep], np.array([len(keep)]), scale)
    assert_close("o", o.cpu().numpy(), ro)
    assert np.max(np.abs(lse.cpu().numpy() - rl)) <= LSE_TOL
    # the hand-off skips (and reports) a block whose page is outside the pool
    pc2 = Paged(B, 4, Hkv, D, spare_pages=0)
    pc2.table[0, 3] = 99
    lg.lg_kv_compact_paged((64, 0, 2**31 - 1, 0), k.cuda(), v.cuda(), *pc2.state())
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) & PAGED_BIT
    written = sorted(pc2.table[0, :3].tolist())
    untouched = [x for x in range(4) if x not in written]
    assert torch.all(pc2.k_pool[untouched].view(torch.int16) == SENTINEL)


def test_broken_append_states_are_reported_and_left_unchanged():
    B, Hkv, D = 1, 2, 64
    kn = torch.zeros(B, Hkv, D, dtype=torch.bfloat16, device="cuda")
    pat = (64, 0, 2**31 - 1, 0)
    # length and position disagree modulo 64
    pc = Paged(B, 2, Hkv, D, spare_pages=0)
    pc.lens.fill_(5)
    pc.pos.fill_(64)
    lg.lg_kv_append_paged(pat, kn, kn, *pc.state())
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) & PAGED_BIT
    assert int(pc.lens) == 5 and int(pc.pos) == 64
    assert torch.all(pc.k_pool.view(torch.int16) == SENTINEL)
    # a full layer with one table entry: the 65th token has no page
    pc = Paged(B, 1, Hkv, D, spare_pages=0)
    for _ in range(64):
        lg.lg_kv_append_paged(pat, kn, kn, *pc.state())
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) == 0
    assert int(pc.lens) == 64 and int(pc.pos) == 64
    lg.lg_kv_append_paged(pat, kn, kn, *pc.state())
    torch.cuda.synchronize()
    assert lg.lg_device_status(0) & PAGED_BIT
    assert int(pc.lens) == 64 and int(pc.pos) == 64
