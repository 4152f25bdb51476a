"""fp64 reference definitions of LongGen masked causal attention (test infrastructure).

Only tests, the smoke check and the bench's CPU-baseline legs use this module;
the CUDA product path never imports it.

Page: "A Little Goes a Long Way: Efficient Long Context Training and Inference
with Partial Contexts" (arXiv 2410.01485).
  * Abstract, insight 1 -- three GPU-friendly sparse patterns: attention sink
    (initial tokens), window attention (recent tokens), blockwise sparse
    attention over strided token blocks.
  * Abstract, insight 2 / atlas.scime.ai summary, "Approach" -- the middle 1/3
    of the layers keep full attention; sparse layers use "static, block-wise
    access"; training uses a FlashAttention-2-based kernel, i.e. exact
    attention.

Readings taken where the pages are silent (each is listed in the design notes):
  * Granularity is block-level: whole ``block_size`` KV blocks are kept, with
    token-level causality (k <= q) as the only token-level term.
  * ``local_blocks`` counts the diagonal block.
  * The strided term is absolute: KV block ``kb`` is kept by every later query
    when ``kb % stride == 0`` (the only reading that lets the sparse layers keep
    a fixed, reduced KV cache).
  * Overlapping terms are a union; scale is explicit (the configs use
    1/sqrt(D)); LSE is the natural log.
  * Decode attends to every cached row of the reduced cache with no mask.

All arithmetic is float64. Arrays use the layouts of the C-ABI:
q, o [B, S, H, D]; k, v [B, S, Hkv, D]; lse [B, H, S]; head h reads KV head
h // (H // Hkv).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

INT32_MAX = 2**31 - 1


@dataclass(frozen=True)
class Pattern:
    """Static block pattern {block_size, sink_blocks, local_blocks, stride}.

    ``stride == 0`` disables the strided term. Full causal attention is
    ``Pattern(b, 0, INT32_MAX, 0)``.
    """

    block_size: int
    sink_blocks: int
    local_blocks: int
    stride: int = 0

    @staticmethod
    def full(block_size: int = 64) -> "Pattern":
        return Pattern(block_size, 0, INT32_MAX, 0)


# ----------------------------------------------------------------------------
# Mask predicate and its block-level view
# ----------------------------------------------------------------------------

def allowed(qi, kj, p: Pattern) -> np.ndarray:
    """Token-level mask: may query token ``qi`` attend to key token ``kj``?

    Causal (kj <= qi) and at least one of: kj's block is a sink block; kj's
    block lies within ``local_blocks`` blocks of qi's block (diagonal included);
    kj's block index is a multiple of ``stride`` (when stride > 0).
    Broadcasts over numpy arrays.
    """
    qi = np.asarray(qi, dtype=np.int64)
    kj = np.asarray(kj, dtype=np.int64)
    qb = qi // p.block_size
    kb = kj // p.block_size
    keep = (kb < p.sink_blocks) | ((qb - kb) < p.local_blocks)
    if p.stride > 0:
        keep = keep | (kb % p.stride == 0)
    return (kj <= qi) & keep


def token_mask(S: int, p: Pattern) -> np.ndarray:
    """The full [S, S] boolean token mask (rows = queries)."""
    q = np.arange(S, dtype=np.int64)[:, None]
    k = np.arange(S, dtype=np.int64)[None, :]
    return allowed(q, k, p)


def _block_occupancy(S: int, p: Pattern) -> np.ndarray:
    """[nqb, nqb] bool: does any allowed token pair fall in block (i, j)?

    Derived by scanning the token mask one query block at a time -- not from a
    block-level formula -- so it pins the block lists to the token predicate.
    """
    b = p.block_size
    if S % b:
        raise ValueError("S must be a multiple of block_size")
    nqb = S // b
    occ = np.zeros((nqb, nqb), dtype=bool)
    keys = np.arange(S, dtype=np.int64)
    for i in range(nqb):
        rows = np.arange(i * b, (i + 1) * b, dtype=np.int64)[:, None]
        m = allowed(rows, keys[None, : (i + 1) * b], p)
        occ[i, : i + 1] = m.reshape(b, i + 1, b).any(axis=(0, 2))
    return occ


def block_lists(S: int, p: Pattern):
    """CSR of KV blocks per query block: (row_ptr[nqb+1], col[nnz]), int32, sorted."""
    occ = _block_occupancy(S, p)
    counts = occ.sum(axis=1)
    row_ptr = np.zeros(occ.shape[0] + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    col = np.nonzero(occ)[1].astype(np.int32)
    return row_ptr, col


def block_lists_t(S: int, p: Pattern):
    """CSC: query blocks per KV block: (col_ptr[nqb+1], row[nnz]), int32, sorted."""
    occ = _block_occupancy(S, p).T
    counts = occ.sum(axis=1)
    col_ptr = np.zeros(occ.shape[0] + 1, dtype=np.int32)
    col_ptr[1:] = np.cumsum(counts)
    row = np.nonzero(occ)[1].astype(np.int32)
    return col_ptr, row


def pair_count(S: int, p: Pattern, chunk: int = 512) -> int:
    """Number of allowed (query, key) token pairs in one head."""
    total = 0
    keys = np.arange(S, dtype=np.int64)[None, :]
    for r0 in range(0, S, chunk):
        rows = np.arange(r0, min(S, r0 + chunk), dtype=np.int64)[:, None]
        total += int(allowed(rows, keys[:, : rows[-1, 0] + 1], p).sum())
    return total


# ----------------------------------------------------------------------------
# Dense formulation (small S): the whole S x S score matrix per head
# ----------------------------------------------------------------------------

def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor
        x = x.detach().to("cpu")
        import torch

        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _masked_softmax(s: np.ndarray, mask: np.ndarray):
    """Row softmax of s over the True entries of mask; returns (P, lse)."""
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(mask, np.exp(s - m), 0.0)
    l = e.sum(axis=-1, keepdims=True)
    lse = (m + np.log(l))[..., 0]
    return e / l, lse


def attention_forward(q, k, v, p: Pattern, scale: float, mask=None):
    """O = softmax_mask(scale * Q K^T) V and LSE per row, dense per head.

    q [B,S,H,D], k/v [B,S,Hkv,D] -> o [B,S,H,D], lse [B,H,S] (natural log).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, H, D = q.shape
    Hkv = k.shape[2]
    g = H // Hkv
    if mask is None:
        mask = token_mask(S, p)
    o = np.zeros((B, S, H, D))
    lse = np.zeros((B, H, S))
    for b in range(B):
        for h in range(H):
            kh = h // g
            s = scale * (q[b, :, h, :] @ k[b, :, kh, :].T)
            P, lse[b, h] = _masked_softmax(s, mask)
            o[b, :, h, :] = P @ v[b, :, kh, :]
    return o, lse


def attention_backward(q, k, v, do, p: Pattern, scale: float, mask=None, o=None):
    """Analytic gradients of sum(O * dO) w.r.t. Q, K, V (dense per head).

    dV = P^T dO;  dP = dO V^T;  Delta = rowsum(P * dP);  dS = P (dP - Delta);
    dQ = scale dS K;  dK = scale dS^T Q.  GQA: dK, dV sum over the query heads
    of a KV group. Returns (dq, dk, dv, delta[B,H,S]).

    With ``o`` given ([B,S,H,D], e.g. the forward output as stored in bf16),
    Delta is taken as rowsum(dO * o) instead -- the identity rowsum(P * dP) =
    dO . O evaluated on the O the backward is handed, which is how a
    FlashAttention-2-style training backward (atlas.scime.ai summary,
    "Approach") forms it. Everything else is unchanged.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    o_in = None if o is None else _f64(o)
    B, S, H, D = q.shape
    Hkv = k.shape[2]
    g = H // Hkv
    if mask is None:
        mask = token_mask(S, p)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    delta = np.zeros((B, H, S))
    for b in range(B):
        for h in range(H):
            kh = h // g
            qh, kk, vv, doh = q[b, :, h], k[b, :, kh], v[b, :, kh], do[b, :, h]
            P, _ = _masked_softmax(scale * (qh @ kk.T), mask)
            dv[b, :, kh] += P.T @ doh
            dP = doh @ vv.T
            if o_in is None:
                delta[b, h] = (P * dP).sum(axis=1)
            else:
                delta[b, h] = (doh * o_in[b, :, h]).sum(axis=1)
            dS = P * (dP - delta[b, h][:, None])
            dq[b, :, h] = scale * (dS @ kk)
            dk[b, :, kh] += scale * (dS.T @ qh)
    return dq, dk, dv, delta


# ----------------------------------------------------------------------------
# Row-gathered formulation (any S): each query row sees only its allowed keys
# ----------------------------------------------------------------------------

def _row_chunks(rows: np.ndarray, chunk: int):
    for i in range(0, len(rows), chunk):
        yield rows[i : i + chunk]


def attention_rows(qh, kh, vh, rows, p: Pattern, scale: float, chunk: int = 64):
    """Forward for selected query rows of ONE head; qh/kh/vh are [S, D].

    Each row's allowed keys are found with the token predicate; masked keys
    contribute nothing, so only those keys are gathered. Returns (o[R,D], lse[R]).
    """
    qh, kh, vh = _f64(qh), _f64(kh), _f64(vh)
    rows = np.asarray(rows, dtype=np.int64)
    o = np.zeros((len(rows), qh.shape[1]))
    lse = np.zeros(len(rows))
    pos = 0
    for r in _row_chunks(rows, chunk):
        keys = np.arange(int(r.max()) + 1, dtype=np.int64)
        m = allowed(r[:, None], keys[None, :], p)
        cols = np.nonzero(m.any(axis=0))[0]
        s = scale * (qh[r] @ kh[cols].T)
        P, l = _masked_softmax(s, m[:, cols])
        o[pos : pos + len(r)] = P @ vh[cols]
        lse[pos : pos + len(r)] = l
        pos += len(r)
    return o, lse


def attention_backward_rows(qh, kh, vh, doh, rows, p: Pattern, scale: float, chunk: int = 64):
    """dQ (and Delta) for selected query rows of one head. Returns (dq[R,D], delta[R])."""
    qh, kh, vh, doh = _f64(qh), _f64(kh), _f64(vh), _f64(doh)
    rows = np.asarray(rows, dtype=np.int64)
    dq = np.zeros((len(rows), qh.shape[1]))
    delta = np.zeros(len(rows))
    pos = 0
    for r in _row_chunks(rows, chunk):
        keys = np.arange(int(r.max()) + 1, dtype=np.int64)
        m = allowed(r[:, None], keys[None, :], p)
        cols = np.nonzero(m.any(axis=0))[0]
        P, _ = _masked_softmax(scale * (qh[r] @ kh[cols].T), m[:, cols])
        dP = doh[r] @ vh[cols].T
        d = (P * dP).sum(axis=1)
        dS = P * (dP - d[:, None])
        dq[pos : pos + len(r)] = scale * (dS @ kh[cols])
        delta[pos : pos + len(r)] = d
        pos += len(r)
    return dq, delta


def attention_backward_kv_rows(qh, kh, vh, doh, krows, p: Pattern, scale: float, chunk: int = 64):
    """dK, dV for selected key rows of one (query head, KV head) pair.

    Every query that may attend to one of ``krows`` contributes; its LSE and
    Delta = dO . O come from its own full forward row. Returns (dk[R,D], dv[R,D]).
    For GQA the caller sums over the query heads of the group.
    """
    qh, kh, vh, doh = _f64(qh), _f64(kh), _f64(vh), _f64(doh)
    S = qh.shape[0]
    krows = np.asarray(krows, dtype=np.int64)
    qall = np.arange(int(krows.min()), S, dtype=np.int64)
    m_all = allowed(qall[:, None], krows[None, :], p)
    qrows = qall[m_all.any(axis=1)]
    m = m_all[m_all.any(axis=1)]
    o, lse = attention_rows(qh, kh, vh, qrows, p, scale, chunk=chunk)
    delta = (doh[qrows] * o).sum(axis=1)
    s = scale * (qh[qrows] @ kh[krows].T)
    P = np.where(m, np.exp(np.where(m, s, 0.0) - lse[:, None]), 0.0)
    dP = doh[qrows] @ vh[krows].T
    dS = P * (dP - delta[:, None])
    dv = P.T @ doh[qrows]
    dk = scale * (dS.T @ qh[qrows])
    return dk, dv


# ----------------------------------------------------------------------------
# Decode over the reduced KV cache, and the split-LSE merge identity
# ----------------------------------------------------------------------------

def decode(q, k_cache, v_cache, cache_lens, scale: float):
    """One-token attention over every cached row (no mask).

    q [B,H,D]; k_cache/v_cache [B,Lmax,Hkv,D]; cache_lens [B] ->
    o [B,H,D], lse [B,H] (natural log).
    """
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    lens = np.asarray(_f64(cache_lens), dtype=np.int64)
    B, H, D = q.shape
    Hkv = kc.shape[2]
    g = H // Hkv
    o = np.zeros((B, H, D))
    lse = np.zeros((B, H))
    for b in range(B):
        n = int(lens[b])
        for h in range(H):
            kk = kc[b, :n, h // g]
            vv = vc[b, :n, h // g]
            s = scale * (kk @ q[b, h])
            m = s.max()
            e = np.exp(s - m)
            l = e.sum()
            lse[b, h] = m + np.log(l)
            o[b, h] = (e @ vv) / l
    return o, lse


def reduced_cache_rows(T: int, p: Pattern) -> np.ndarray:
    """Prompt rows the reduced KV cache of a sparse layer holds when decoding
    the token at position T: every key token kj < T that query T may attend
    (Abstract: "GPU-friendly KV cache reduction"; the cache keeps only what
    the static pattern can still reach), ascending. int64 row indices."""
    kj = np.arange(T, dtype=np.int64)
    return kj[allowed(T, kj, p)]


def reduced_cache(k, v, T: int, p: Pattern):
    """Gather the reduced cache from prompt K/V [B, >=T, Hkv, D]: returns
    (k_cache [B, n, Hkv, D], v_cache [B, n, Hkv, D], rows [n]) with the rows of
    ``reduced_cache_rows`` in that order (values copied, not converted)."""
    rows = reduced_cache_rows(T, p)
    k = np.asarray(k)
    v = np.asarray(v)
    return k[:, rows], v[:, rows], rows


def merge_partials(o_parts, lse_parts):
    """Combine attention over disjoint key subsets: lse = log sum exp(lse_s),
    o = sum_s exp(lse_s - lse) o_s. Empty parts carry lse_s = -inf."""
    o_parts = _f64(o_parts)
    lse_parts = _f64(lse_parts)
    live = np.isfinite(lse_parts)
    m = np.max(lse_parts[live])
    lse = m + np.log(np.exp(lse_parts[live] - m).sum())
    w = np.where(live, np.exp(np.where(live, lse_parts, 0.0) - lse), 0.0)
    o = (w[:, None] * np.where(live[:, None], o_parts, 0.0)).sum(axis=0)
    return o, lse
