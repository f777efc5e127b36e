"""Plain fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or helper with the CUDA library; the only thing both sides use
is the seeded input generator, which holds none of the method's arithmetic.

What it computes (the definition, written out, nothing more):

* Forward.  For every batch b and query head h (key/value head
  ``h // (Hq // Hkv)``), ``S = scale * Q K^T`` over all N keys, the causal mask
  sets ``S[i, j] = -inf`` for ``j > i``, every row of ``S`` is turned into a
  probability vector by the full (materialised) softmax, ``O = P V`` and
  ``lse[i] = log(sum_j exp(S[i, j]))`` (natural log of the scaled, masked
  scores).  The pages state that every FlashAttention generation keeps "the
  same exact attention math" (r/mlscaling, FlashAttention-PyTorch post, list
  of FA1-FA4); this is that math, with no tiling, no online recurrence and no
  deferred normalisation.
* Backward.  The plain softmax Jacobian: ``dV = P^T dO``, ``dP = dO V^T``,
  ``dS[i, j] = P[i, j] (dP[i, j] - sum_k P[i, k] dP[i, k])``,
  ``dQ = scale dS K``, ``dK = scale dS^T Q``; for grouped-query attention dK
  and dV are summed over the query heads that share a key/value head.  The
  recompute-from-saved-statistics backward named on the pages
  (FlashAttention (Metal Port) README, Documentation section: the backward
  pass with its GEMMs and scratch for partial sums) reaches the same numbers;
  this oracle does not use the shortcut ``rowsum(dO * O)`` for the row term,
  it sums ``P * dP`` directly.

Readings where the pages are silent (the plainest ones the rest supports): top-left
causal alignment with equal query and key lengths; contiguous GQA groups
(query head h reads key/value head ``h // G``); lse in natural log.

Local (sliding-window) attention, the mask variant the pages mention
(FlashAttention entity page and heapsort-ai.news attention tag: global plus
sliding-window attention; twiscan MHA search: a 112-token local window):
``window=(wl, wr)`` lets query i see key j only when ``i - wl <= j <= i + wr``;
a negative bound is unbounded on that side.  ``causal`` is the same as
``window=(-1, 0)`` and both may be combined.

Block-sparse attention, the other mask variant the pages name (FlashAttention
(Metal Port) README, Documentation section: block sparsity as a customisation
of the basic algorithm; FlashPrefill V2 finding on the FlashAttention entity
page: block-sparse prefill): ``block_mask`` [B, Hq, T, T] (T = ceil(N / block))
lets query i see key j only when ``block_mask[b, h, i // block, j // block]``
is nonzero, on top of the causal/window mask.  A query row that sees no key
at all has ``O = 0`` and ``lse = -inf`` (its softmax has no terms) and passes
no gradient.

Precision: every input is upcast to float64 first; numpy/OpenBLAS does the
matrix products (a library primitive used as one step, no fusion).
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "attention_fwd",
    "attention_bwd",
    "attention_fwd_rows",
    "attention_decode",
    "softmax_probs",
]

# Largest number of query rows whose full score rows are materialised at once.
# Only bounds host memory; the result does not depend on it.
_ROW_BLOCK = 1024


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _check_shapes(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, H, N, D]")
    b, hq, n, d = q.shape
    if k.shape != v.shape or k.shape[0] != b or k.shape[2] != n or k.shape[3] != d:
        raise ValueError(f"shape mismatch q{q.shape} k{k.shape} v{v.shape}")
    hkv = k.shape[1]
    if hkv < 1 or hq % hkv != 0:
        raise ValueError(f"Hq={hq} is not a multiple of Hkv={hkv}")
    return b, hq, hkv, n, d


def _scores(q_rows: np.ndarray, k_all: np.ndarray, row_ids: np.ndarray,
            causal: bool, scale: float, window=None, block_mask=None,
            block: int = 128) -> np.ndarray:
    """Scaled, masked scores for the given query rows against every key.

    ``block_mask``: this (batch, head)'s [T, T] tile mask, or None."""
    s = scale * (q_rows @ k_all.T)
    cols = np.arange(k_all.shape[0])[None, :]
    rows = row_ids[:, None]
    if causal:
        s = np.where(cols > rows, -np.inf, s)
    if window is not None:
        wl, wr = window
        if wl >= 0:
            s = np.where(cols < rows - wl, -np.inf, s)
        if wr >= 0:
            s = np.where(cols > rows + wr, -np.inf, s)
    if block_mask is not None:
        bm = np.asarray(block_mask) != 0
        allowed = bm[row_ids // block][:, np.arange(k_all.shape[0]) // block]
        s = np.where(allowed, s, -np.inf)
    return s


def softmax_probs(s: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Full-row softmax of a score block; returns (P, lse) with lse natural-log.

    A row whose scores are all -inf (no visible key) gets P = 0, lse = -inf."""
    m = np.max(s, axis=1, keepdims=True)
    empty = ~np.isfinite(m)
    e = np.exp(s - np.where(empty, 0.0, m))
    z = np.sum(e, axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(empty, 0.0, e / np.where(empty, 1.0, z))
        lse = np.where(empty, -np.inf, m + np.log(np.where(empty, 1.0, z)))[:, 0]
    return p, lse


def _bm(block_mask, b, h):
    return None if block_mask is None else np.asarray(block_mask)[b, h]


def attention_fwd(q, k, v, causal: bool, scale: float, window=None, block_mask=None,
                  block: int = 128):
    """O [B,Hq,N,D] and lse [B,Hq,N] in float64 for the whole problem."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    b_, hq, hkv, n, d = _check_shapes(q, k, v)
    g = hq // hkv
    o = np.empty((b_, hq, n, d), dtype=np.float64)
    lse = np.empty((b_, hq, n), dtype=np.float64)
    for b in range(b_):
        for h in range(hq):
            hk = h // g
            for r0 in range(0, n, _ROW_BLOCK):
                rows = np.arange(r0, min(n, r0 + _ROW_BLOCK))
                s = _scores(q[b, h, rows], k[b, hk], rows, causal, scale, window,
                            _bm(block_mask, b, h), block)
                p, l = softmax_probs(s)
                o[b, h, rows] = p @ v[b, hk]
                lse[b, h, rows] = l
    return o, lse


def attention_fwd_rows(q, k, v, causal: bool, scale: float, b: int, h: int, rows, window=None,
                       block_mask=None, block: int = 128):
    """O and lse of selected query rows of one (batch, query head) only.

    Rows of attention are independent, so this is the same definition
    restricted to a subset; it lets parity tests at full problem sizes check
    sampled rows without materialising every score row.
    """
    hq, hkv = q.shape[1], k.shape[1]
    hk = h // (hq // hkv)
    rows = np.asarray(rows, dtype=np.int64)
    qr = _f64(q[b, h][rows])
    kk = _f64(k[b, hk])
    vv = _f64(v[b, hk])
    s = _scores(qr, kk, rows, causal, scale, window, _bm(block_mask, b, h), block)
    p, l = softmax_probs(s)
    return p @ vv, l


def attention_bwd(q, k, v, do, causal: bool, scale: float, heads=None, window=None,
                  block_mask=None, block: int = 128):
    """(dQ, dK, dV) in float64 from the plain softmax Jacobian.

    ``heads``: optional iterable of (b, h_kv) pairs to restrict the work to
    (the other entries of the outputs are left as NaN); every query head of
    each listed key/value group is included, so the listed dK/dV are complete.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    b_, hq, hkv, n, d = _check_shapes(q, k, v)
    if do.shape != q.shape:
        raise ValueError("dO must have the shape of Q")
    g = hq // hkv
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    pairs = [(b, hk) for b in range(b_) for hk in range(hkv)] if heads is None else list(heads)
    for b, hk in pairs:
        dk_acc = np.zeros((n, d))
        dv_acc = np.zeros((n, d))
        for h in range(hk * g, (hk + 1) * g):
            dq_h = np.empty((n, d))
            for r0 in range(0, n, _ROW_BLOCK):
                rows = np.arange(r0, min(n, r0 + _ROW_BLOCK))
                s = _scores(q[b, h, rows], k[b, hk], rows, causal, scale, window,
                            _bm(block_mask, b, h), block)
                p, _ = softmax_probs(s)
                dO = do[b, h, rows]
                dv_acc += p.T @ dO
                dp = dO @ v[b, hk].T
                row_term = np.sum(p * dp, axis=1, keepdims=True)
                ds = p * (dp - row_term)
                dq_h[rows] = scale * (ds @ k[b, hk])
                dk_acc += scale * (ds.T @ q[b, h, rows])
            dq[b, h] = dq_h
        dk[b, hk] = dk_acc
        dv[b, hk] = dv_acc
    return dq, dk, dv


def attention_decode(q, k_pool, v_pool, block_table, seqlens, causal: bool, scale: float,
                     page: int = 128):
    """Attention of a few new query tokens against a paged key/value cache.

    The decode step the pages pair with paged KV caches (FlashPrefill V2 and
    vLLM findings on the FlashAttention entity page: paged KV cache,
    continuous batching), written out plainly:

    * ``q`` [B, Hq, Sq, D]: the Sq newest tokens of each sequence b;
    * ``k_pool``, ``v_pool`` [P, page, Hkv, D]: the cache pages; sequence b
      holds its ``seqlens[b]`` keys in pages ``block_table[b][0..]`` (key t
      of the sequence is row ``t % page`` of page ``block_table[b][t // page]``);
    * query token i of sequence b sits at position ``seqlens[b] - Sq + i``;
      causal lets it see keys at positions <= its own, otherwise it sees all
      ``seqlens[b]`` keys; a token that sees no key gets O = 0, lse = -inf.

    Returns O [B, Hq, Sq, D] and lse [B, Hq, Sq] (natural log) in float64.
    """
    q = _f64(q)
    kp, vp = _f64(k_pool), _f64(v_pool)
    b_, hq, sq, d = q.shape
    hkv = kp.shape[2]
    g = hq // hkv
    o = np.zeros((b_, hq, sq, d))
    lse = np.full((b_, hq, sq), -np.inf)
    for b in range(b_):
        n = int(seqlens[b])
        t = np.arange(n)
        pages = np.asarray(block_table[b])[t // page]
        kk = kp[pages, t % page]  # [n, Hkv, D]
        vv = vp[pages, t % page]
        pos = n - sq + np.arange(sq)
        for h in range(hq):
            hk = h // g
            s = scale * (q[b, h] @ kk[:, hk].T) if n else np.zeros((sq, 0))
            if causal:
                s = np.where(t[None, :] > pos[:, None], -np.inf, s)
            if n == 0:
                continue
            p, l = softmax_probs(s)
            o[b, h] = p @ vv[:, hk]
            lse[b, h] = l
    return o, lse
