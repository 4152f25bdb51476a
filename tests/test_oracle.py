"""Pins for the fp64 oracle, checked against things other than itself.

Each pin ties one oracle function to something independent of its code:
  * hand-derived closed-form block and pair counts (tests/golden/pattern_counts.txt);
  * torch's float64 scaled_dot_product_attention and autograd (library routines)
    on the special cases where the pattern reduces to plain causal attention,
    block-diagonal attention, or attention over explicitly gathered key blocks;
  * closed forms (constant keys give the mean of the visible values; all-ones
    values give ones);
  * central finite differences of L = sum(O * dO) for the gradients;
  * the split-LSE merge identity and the decode/prefill row identity.
The last group plants mistakes in a copy of the oracle and checks that a pin
catches each one.
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import Pattern
from oracle import attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pattern_counts.txt")


def load_golden():
    rows = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, S, b, sink, local, stride, nnz, pairs = line.split()
            rows[name] = (int(S), Pattern(int(b), int(sink), int(local), int(stride)), int(nnz), int(pairs))
    return rows


def rnd(shape, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape)


def sdpa64(q, k, v, mask=None, causal=False, scale=None):
    """torch SDPA in float64 on [L, D] single-head arrays."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x))[None, None] for x in (q, k, v))
    am = None if mask is None else torch.from_numpy(mask)[None, None]
    out = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=am, is_causal=causal, scale=scale)
    return out[0, 0].numpy()


# ----------------------------------------------------------------------------
# Pattern: hand-derived counts
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["c1_sink_local4", "c3_analog_4096"])
def test_block_lists_match_hand_counts(name):
    S, p, nnz, pairs = load_golden()[name]
    row_ptr, col = oracle.block_lists(S, p)
    assert int(row_ptr[-1]) == nnz == len(col)
    assert oracle.pair_count(S, p) == pairs
    col_ptr, row = oracle.block_lists_t(S, p)
    assert int(col_ptr[-1]) == nnz


@pytest.mark.parametrize("name", ["c2_sink_window", "c2_dense"])
def test_pair_counts_32k_match_hand_counts(name):
    S, p, nnz, pairs = load_golden()[name]
    assert oracle.pair_count(S, p, chunk=1024) == pairs


def test_c1_block_list_contents():
    # {64,1,4,0}: block 0 (sink) plus blocks i-3..i (the diagonal is local).
    S, p, _, _ = load_golden()["c1_sink_local4"]
    row_ptr, col = oracle.block_lists(S, p)
    for i in range(S // 64):
        expect = sorted({0} | set(range(max(0, i - 3), i + 1)))
        assert col[row_ptr[i]:row_ptr[i + 1]].tolist() == expect


def test_transpose_is_transpose():
    p = Pattern(16, 2, 3, 5)
    S = 16 * 40
    row_ptr, col = oracle.block_lists(S, p)
    col_ptr, row = oracle.block_lists_t(S, p)
    a = {(i, int(j)) for i in range(S // 16) for j in col[row_ptr[i]:row_ptr[i + 1]]}
    b = {(int(i), j) for j in range(S // 16) for i in row[col_ptr[j]:col_ptr[j + 1]]}
    assert a == b


# ----------------------------------------------------------------------------
# Forward: special cases that reduce to library attention
# ----------------------------------------------------------------------------

def test_full_pattern_is_causal_sdpa():
    S, D, scale = 256, 16, 0.37
    q, k, v = rnd((1, S, 2, D), 1), rnd((1, S, 2, D), 2), rnd((1, S, 2, D), 3)
    o, lse = oracle.attention_forward(q, k, v, Pattern.full(16), scale)
    for h in range(2):
        ref = sdpa64(q[0, :, h], k[0, :, h], v[0, :, h], causal=True, scale=scale)
        np.testing.assert_allclose(o[0, :, h], ref, atol=1e-12, rtol=0)
        s = scale * q[0, :, h] @ k[0, :, h].T
        s[np.triu_indices(S, 1)] = -np.inf
        np.testing.assert_allclose(lse[0, h], torch.logsumexp(torch.from_numpy(s), dim=1).numpy(), atol=1e-12)


def test_window_covering_sequence_is_full():
    S, D = 192, 8
    q, k, v = rnd((1, S, 1, D), 4), rnd((1, S, 1, D), 5), rnd((1, S, 1, D), 6)
    a, la = oracle.attention_forward(q, k, v, Pattern(16, 0, S // 16, 0), 0.5)
    b, lb = oracle.attention_forward(q, k, v, Pattern.full(16), 0.5)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)


def test_single_local_block_is_blockwise_causal():
    bs, nb, D = 16, 6, 8
    S = bs * nb
    q, k, v = rnd((1, S, 1, D), 7), rnd((1, S, 1, D), 8), rnd((1, S, 1, D), 9)
    o, _ = oracle.attention_forward(q, k, v, Pattern(bs, 0, 1, 0), 0.3)
    for i in range(nb):
        sl = slice(i * bs, (i + 1) * bs)
        ref = sdpa64(q[0, sl, 0], k[0, sl, 0], v[0, sl, 0], causal=True, scale=0.3)
        np.testing.assert_allclose(o[0, sl, 0], ref, atol=1e-12)


def gathered_reference(q, k, v, bs, blocks_of, scale):
    """Attention per query block over an explicitly gathered key-block set;
    blocks strictly below the diagonal are fully visible, the diagonal block is
    causal (torch float64 SDPA with a tril mask on the diagonal part)."""
    S, D = q.shape
    out = np.zeros_like(q)
    for i in range(S // bs):
        blocks = sorted(blocks_of(i))
        assert blocks[-1] == i
        keys = np.concatenate([np.arange(j * bs, (j + 1) * bs) for j in blocks])
        mask = np.ones((bs, len(keys)), dtype=bool)
        mask[:, -bs:] = np.tril(np.ones((bs, bs), dtype=bool))
        sl = slice(i * bs, (i + 1) * bs)
        out[sl] = sdpa64(q[sl], k[keys], v[keys], mask=mask, scale=scale)
    return out


@pytest.mark.parametrize("p", [Pattern(16, 1, 1, 0), Pattern(16, 2, 3, 0), Pattern(16, 0, 1, 4),
                               Pattern(16, 1, 4, 0), Pattern(16, 1, 2, 3)])
def test_patterns_match_gathered_sdpa(p):
    bs, nb, D, scale = 16, 13, 8, 0.41
    S = bs * nb
    q, k, v = rnd((1, S, 1, D), 10), rnd((1, S, 1, D), 11), rnd((1, S, 1, D), 12)
    o, _ = oracle.attention_forward(q, k, v, p, scale)

    def blocks_of(i):
        sink = set(range(min(p.sink_blocks, i + 1)))
        window = set(range(max(0, i - p.local_blocks + 1), i + 1))
        strided = set(range(0, i + 1, p.stride)) if p.stride else set()
        return sink | window | strided

    ref = gathered_reference(q[0, :, 0], k[0, :, 0], v[0, :, 0], bs, blocks_of, scale)
    np.testing.assert_allclose(o[0, :, 0], ref, atol=1e-12)


def test_gqa_equals_repeated_kv():
    S, D = 128, 8
    q = rnd((2, S, 4, D), 13)
    k, v = rnd((2, S, 2, D), 14), rnd((2, S, 2, D), 15)
    p = Pattern(16, 1, 2, 3)
    o1, l1 = oracle.attention_forward(q, k, v, p, 0.3)
    o2, l2 = oracle.attention_forward(q, np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2), p, 0.3)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_closed_forms_constant_keys_and_unit_values():
    bs, S, D = 8, 64, 4
    p = Pattern(bs, 1, 2, 3)
    q = rnd((1, S, 1, D), 16)
    k = np.ones((1, S, 1, D))
    v = rnd((1, S, 1, D), 17)
    o, lse = oracle.attention_forward(q, k, v, p, 0.7)
    mask = oracle.token_mask(S, p)
    for i in range(S):
        vis = np.nonzero(mask[i])[0]
        np.testing.assert_allclose(o[0, i, 0], v[0, vis, 0].mean(axis=0), atol=1e-13)
        np.testing.assert_allclose(lse[0, 0, i], 0.7 * q[0, i, 0].sum() + math.log(len(vis)), atol=1e-12)
    o1, _ = oracle.attention_forward(q, rnd((1, S, 1, D), 18), np.ones((1, S, 1, D)), p, 0.7)
    np.testing.assert_allclose(o1, 1.0, atol=1e-13)


@pytest.mark.parametrize("p", [Pattern(16, 1, 3, 0), Pattern(16, 1, 2, 4), Pattern.full(16)])
def test_row_gathered_matches_dense(p):
    S, D = 320, 16
    q, k, v = rnd((S, D), 19), rnd((S, D), 20), rnd((S, D), 21)
    o, lse = oracle.attention_forward(q[None, :, None], k[None, :, None], v[None, :, None], p, 0.25)
    rows = np.array([0, 1, 15, 16, 17, 100, 255, 256, 319])
    o2, l2 = oracle.attention_rows(q, k, v, rows, p, 0.25, chunk=4)
    np.testing.assert_allclose(o2, o[0, rows, 0], atol=1e-13)
    np.testing.assert_allclose(l2, lse[0, 0, rows], atol=1e-13)


def test_row_gathered_full_matches_sdpa_2k():
    S, D = 2048, 32
    q, k, v = rnd((S, D), 22), rnd((S, D), 23), rnd((S, D), 24)
    rows = np.array([0, 7, 1000, 2047])
    o, _ = oracle.attention_rows(q, k, v, rows, Pattern.full(64), 0.2)
    ref = sdpa64(q, k, v, causal=True, scale=0.2)
    np.testing.assert_allclose(o, ref[rows], atol=1e-12)


# ----------------------------------------------------------------------------
# Backward
# ----------------------------------------------------------------------------

def loss(q, k, v, do, p, scale):
    o, _ = oracle.attention_forward(q, k, v, p, scale)
    return float((o * do).sum())


def test_gradients_central_differences():
    S, D, scale = 48, 4, 0.6
    p = Pattern(8, 1, 2, 3)
    q, k, v, do = rnd((1, S, 2, D), 25), rnd((1, S, 1, D), 26), rnd((1, S, 1, D), 27), rnd((1, S, 2, D), 28)
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, p, scale)
    h = 1e-6
    rng = np.random.default_rng(29)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            fp = loss(**{**args, name: xp}, do=do, p=p, scale=scale)
            fm = loss(**{**args, name: xm}, do=do, p=p, scale=scale)
            fd = (fp - fm) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(g[idx])), (name, idx, fd, g[idx])


@pytest.mark.parametrize("p", [Pattern(16, 1, 4, 0), Pattern(16, 0, 2, 3), Pattern.full(16)])
def test_gradients_match_torch_autograd(p):
    S, D, scale = 160, 8, 0.35
    q, k, v, do = (rnd((S, D), s) for s in (30, 31, 32, 33))
    dq, dk, dv, delta = oracle.attention_backward(q[None, :, None], k[None, :, None], v[None, :, None],
                                                  do[None, :, None], p, scale)
    tq, tk, tv = (torch.from_numpy(x.copy()).requires_grad_(True) for x in (q, k, v))
    mask = torch.from_numpy(oracle.token_mask(S, p))
    out = F.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None],
                                         attn_mask=mask[None, None], scale=scale)[0, 0]
    (out * torch.from_numpy(do)).sum().backward()
    np.testing.assert_allclose(dq[0, :, 0], tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk[0, :, 0], tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv[0, :, 0], tv.grad.numpy(), atol=1e-12)
    # Delta = rowsum(P * dP) equals dO . O
    np.testing.assert_allclose(delta[0, 0], (out.detach().numpy() * do).sum(axis=1), atol=1e-12)


def test_gradients_with_given_output_follow_its_delta():
    """Delta from a given O: with the exact O the gradients are the autograd-pinned
    ones (Delta = dO . O); with a perturbed O, Delta is rowsum(dO * O_given), and
    dV (which has no Delta term) does not move while dQ and dK do."""
    S, D, scale = 96, 8, 0.35
    p = Pattern(16, 1, 2, 3)
    q, do = rnd((1, S, 2, D), 50), rnd((1, S, 2, D), 51)
    k, v = rnd((1, S, 1, D), 52), rnd((1, S, 1, D), 53)
    o, _ = oracle.attention_forward(q, k, v, p, scale)
    ref = oracle.attention_backward(q, k, v, do, p, scale)
    got = oracle.attention_backward(q, k, v, do, p, scale, o=o)
    for a, b in zip(ref, got):
        np.testing.assert_allclose(a, b, atol=1e-12)
    o2 = o + 0.01 * rnd(o.shape, 54)
    dq2, dk2, dv2, delta2 = oracle.attention_backward(q, k, v, do, p, scale, o=o2)
    np.testing.assert_allclose(delta2, np.einsum("bshd,bshd->bhs", do, o2), atol=1e-12)
    np.testing.assert_allclose(dv2, ref[2], atol=1e-12)
    assert np.abs(dq2 - ref[0]).max() > 1e-4 and np.abs(dk2 - ref[1]).max() > 1e-4


def test_gqa_gradients_sum_over_group():
    S, D = 96, 8
    p = Pattern(16, 1, 2, 0)
    q, do = rnd((1, S, 4, D), 34), rnd((1, S, 4, D), 35)
    k, v = rnd((1, S, 2, D), 36), rnd((1, S, 2, D), 37)
    dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, p, 0.4)
    dq2, dk2, dv2, _ = oracle.attention_backward(q, np.repeat(k, 2, 2), np.repeat(v, 2, 2), do, p, 0.4)
    np.testing.assert_allclose(dq, dq2, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(1, S, 2, 2, D).sum(3), atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(1, S, 2, 2, D).sum(3), atol=1e-13)


@pytest.mark.parametrize("p", [Pattern(16, 1, 3, 0), Pattern(16, 1, 2, 4)])
def test_row_gathered_backward_matches_dense(p):
    S, D, scale = 256, 8, 0.3
    q, k, v, do = (rnd((S, D), s) for s in (38, 39, 40, 41))
    dq, dk, dv, delta = oracle.attention_backward(q[None, :, None], k[None, :, None], v[None, :, None],
                                                  do[None, :, None], p, scale)
    rows = np.array([0, 5, 16, 64, 130, 255])
    dq_r, d_r = oracle.attention_backward_rows(q, k, v, do, rows, p, scale, chunk=4)
    np.testing.assert_allclose(dq_r, dq[0, rows, 0], atol=1e-13)
    np.testing.assert_allclose(d_r, delta[0, 0, rows], atol=1e-13)
    krows = np.array([0, 1, 15, 33, 64, 200, 255])
    dk_r, dv_r = oracle.attention_backward_kv_rows(q, k, v, do, krows, p, scale, chunk=16)
    np.testing.assert_allclose(dk_r, dk[0, krows, 0], atol=1e-13)
    np.testing.assert_allclose(dv_r, dv[0, krows, 0], atol=1e-13)


# ----------------------------------------------------------------------------
# Decode and the split merge
# ----------------------------------------------------------------------------

def test_decode_matches_sdpa_ragged():
    B, H, Hkv, D, L = 3, 4, 2, 16, 50
    q, kc, vc = rnd((B, H, D), 42), rnd((B, L, Hkv, D), 43), rnd((B, L, Hkv, D), 44)
    lens = np.array([50, 1, 23])
    o, lse = oracle.decode(q, kc, vc, lens, 0.25)
    for b in range(B):
        for h in range(H):
            n = lens[b]
            ref = sdpa64(q[b, h][None], kc[b, :n, h // 2], vc[b, :n, h // 2], scale=0.25)
            np.testing.assert_allclose(o[b, h], ref[0], atol=1e-13)
            s = torch.from_numpy(0.25 * kc[b, :n, h // 2] @ q[b, h])
            assert abs(lse[b, h] - torch.logsumexp(s, 0).item()) < 1e-12


def test_decode_over_gathered_cache_equals_prefill_row():
    p = Pattern(16, 1, 3, 4)
    S, D, scale = 16 * 20, 8, 0.3
    q, k, v = rnd((S, D), 45), rnd((S, D), 46), rnd((S, D), 47)
    for row in (0, 17, 150, 319):
        keys = np.nonzero(oracle.allowed(row, np.arange(S), p))[0]
        perm = np.random.default_rng(row).permutation(len(keys))  # ring order is irrelevant
        kc, vc = k[keys][perm], v[keys][perm]
        o, lse = oracle.decode(q[row][None, None], kc[None, :, None], vc[None, :, None], [len(keys)], scale)
        o2, l2 = oracle.attention_rows(q, k, v, [row], p, scale)
        np.testing.assert_allclose(o[0, 0], o2[0], atol=1e-13)
        assert abs(lse[0, 0] - l2[0]) < 1e-12


GOLDEN_CACHE = os.path.join(os.path.dirname(__file__), "golden", "reduced_cache_rows.txt")


def load_cache_golden():
    rows = {}
    with open(GOLDEN_CACHE) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, T, b, sink, local, stride, n = line.split()
            rows[name] = (int(T), Pattern(int(b), int(sink), int(local), int(stride)), int(n))
    return rows


@pytest.mark.parametrize("name", sorted(load_cache_golden()))
def test_reduced_cache_rows_match_hand_counts(name):
    T, p, n = load_cache_golden()[name]
    rows = oracle.reduced_cache_rows(T, p)
    assert len(rows) == n
    assert np.all(np.diff(rows) > 0) and (n == 0 or rows[-1] < T)


@pytest.mark.parametrize("p", [Pattern(16, 1, 3, 4), Pattern(16, 2, 2, 0), Pattern(16, 0, 1, 0), Pattern.full(16)])
def test_decode_over_reduced_cache_plus_own_row_equals_prefill_row(p):
    # The hand-off identity: decoding token T over the reduced cache of the
    # prompt [0, T) plus its own K/V row gives prefill attention row T.
    S, D, scale = 16 * 12, 8, 0.3
    q, k, v = rnd((S, D), 60), rnd((S, D), 61), rnd((S, D), 62)
    for T in (16, 80, 176):
        kc, vc, rows = oracle.reduced_cache(k[None, :, None], v[None, :, None], T, p)
        kc = np.concatenate([kc, k[None, T:T + 1, None]], axis=1)
        vc = np.concatenate([vc, v[None, T:T + 1, None]], axis=1)
        o, lse = oracle.decode(q[T][None, None], kc, vc, [kc.shape[1]], scale)
        o2, l2 = oracle.attention_rows(q, k, v, [T], p, scale)
        np.testing.assert_allclose(o[0, 0], o2[0], atol=1e-13)
        assert abs(lse[0, 0] - l2[0]) < 1e-12


@pytest.mark.parametrize("nsplit", [1, 2, 5, 17])
def test_merge_of_any_partition_equals_unsplit(nsplit):
    L, D = 97, 8
    q, kc, vc = rnd((1, 1, D), 48), rnd((1, L, 1, D), 49), rnd((1, L, 1, D), 50)
    o, lse = oracle.decode(q, kc, vc, [L], 0.5)
    cuts = np.sort(np.random.default_rng(nsplit).choice(np.arange(1, L), nsplit - 1, replace=False))
    bounds = np.concatenate([[0], cuts, [L]])
    parts_o, parts_l = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        po, pl = oracle.decode(q, kc[:, a:b], vc[:, a:b], [b - a], 0.5)
        parts_o.append(po[0, 0])
        parts_l.append(pl[0, 0])
    parts_o.append(np.full(D, np.nan))  # an empty split
    parts_l.append(-np.inf)
    mo, ml = oracle.merge_partials(np.array(parts_o), np.array(parts_l))
    np.testing.assert_allclose(mo, o[0, 0], atol=1e-12)
    assert abs(ml - lse[0, 0]) < 1e-12


# ----------------------------------------------------------------------------
# Planted mistakes: each must be caught by one of the pins above
# ----------------------------------------------------------------------------

def test_pins_catch_planted_mask_mistakes(monkeypatch):
    S, p, nnz, pairs = load_golden()["c1_sink_local4"]
    real = oa.allowed

    def off_by_one_window(qi, kj, pp):
        qi = np.asarray(qi); kj = np.asarray(kj)
        qb, kb = qi // pp.block_size, kj // pp.block_size
        return (kj <= qi) & ((kb < pp.sink_blocks) | ((qb - kb) <= pp.local_blocks))

    def no_causality(qi, kj, pp):
        qi = np.asarray(qi); kj = np.asarray(kj)
        return real(np.maximum(qi, kj), kj, pp)

    def relative_stride(qi, kj, pp):
        qi = np.asarray(qi); kj = np.asarray(kj)
        qb, kb = qi // pp.block_size, kj // pp.block_size
        keep = (kb < pp.sink_blocks) | ((qb - kb) < pp.local_blocks) | ((qb - kb) % 32 == 0)
        return (kj <= qi) & keep

    for bad in (off_by_one_window, no_causality):
        monkeypatch.setattr(oa, "allowed", bad)
        assert oa.pair_count(S, p) != pairs
    monkeypatch.setattr(oa, "allowed", relative_stride)
    S3, p3, nnz3, pairs3 = load_golden()["c3_analog_4096"]
    assert oa.pair_count(S3, p3) != pairs3


def causal_sdpa_error():
    S, D, scale = 128, 8, 0.37
    q, k, v = rnd((1, S, 1, D), 1), rnd((1, S, 1, D), 2), rnd((1, S, 1, D), 3)
    o, _ = oracle.attention_forward(q, k, v, Pattern.full(16), scale)
    return np.abs(o[0, :, 0] - sdpa64(q[0, :, 0], k[0, :, 0], v[0, :, 0], causal=True, scale=scale)).max()


def fd_error(backward):
    """Max |finite difference - analytic| over a few sampled entries."""
    S, D, scale = 32, 4, 0.6
    p = Pattern(8, 1, 2, 0)
    q, k, v, do = rnd((1, S, 1, D), 55), rnd((1, S, 1, D), 56), rnd((1, S, 1, D), 57), rnd((1, S, 1, D), 58)
    grads = backward(q, k, v, do, p, scale)
    rng = np.random.default_rng(59)
    err = 0.0
    for xi, name in enumerate(("q", "k", "v")):
        for _ in range(6):
            args = {"q": q, "k": k, "v": v}
            idx = tuple(int(rng.integers(0, n)) for n in q.shape)
            xp, xm = args[name].copy(), args[name].copy()
            xp[idx] += 1e-6
            xm[idx] -= 1e-6
            fd = (loss(**{**args, name: xp}, do=do, p=p, scale=scale)
                  - loss(**{**args, name: xm}, do=do, p=p, scale=scale)) / 2e-6
            err = max(err, abs(fd - grads[xi][idx]))
    return err


def test_pins_catch_planted_forward_mistake(monkeypatch):
    assert causal_sdpa_error() < 1e-12
    real_softmax = oa._masked_softmax
    monkeypatch.setattr(oa, "_masked_softmax", lambda s, m: real_softmax(1.5 * s, m))  # scale applied twice
    assert causal_sdpa_error() > 1e-3


def test_pins_catch_planted_gradient_mistakes():
    assert fd_error(oracle.attention_backward) < 1e-7

    def dropped_delta(q, k, v, do, p, scale):  # plant: dS = P * dP (Delta term dropped)
        qh, kh, vh, doh = q[0, :, 0], k[0, :, 0], v[0, :, 0], do[0, :, 0]
        P, _ = oa._masked_softmax(scale * qh @ kh.T, oracle.token_mask(qh.shape[0], p))
        dS = P * (doh @ vh.T)
        return ((scale * dS @ kh)[None, :, None], (scale * dS.T @ qh)[None, :, None],
                (P.T @ doh)[None, :, None])

    def transposed_dv(q, k, v, do, p, scale):  # plant: dV = P dO instead of P^T dO
        dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, p, scale)
        P, _ = oa._masked_softmax(scale * q[0, :, 0] @ k[0, :, 0].T, oracle.token_mask(q.shape[1], p))
        return dq, dk, (P @ do[0, :, 0])[None, :, None]

    assert fd_error(dropped_delta) > 1e-3
    assert fd_error(transposed_dv) > 1e-3
