"""Plain fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
module.  The product path (the CUDA library and its Python binding) never
imports or calls it, and this module imports nothing from the product.

What it computes, and where the pages define it
-----------------------------------------------
Sources (web pages on FlashAttention; cited by page title and section):

* "Flash Attention" (karlkratz.de), sections "Tiling: Blockweise Berechnung im
  schnellen Speicher", "Speicherbedarf und Laufzeitverhalten",
  "Recomputation beim Rückwärtsdurchlauf".
* "Flash Attention" (Ultralytics glossary), sections "Принцип работы Flash
  Attention" (algorithm description and the PyTorch demonstration with its
  printed error) and "Flash Attention и смежные понятия" (standard attention).

Both pages state that the tiled method computes *exactly* standard attention
(up to floating-point rounding), so the oracle is the plain definition written
out, materialising the full score matrix S and probability matrix P per
(batch, head) in float64:

    S_ij  = scale * <q_i, k_j>            (-inf where j > i when causal)
    m_i   = max_j S_ij
    P_ij  = exp(S_ij - m_i) / sum_j exp(S_ij - m_i)
    O_i   = sum_j P_ij v_j
    LSE_i = m_i + ln sum_j exp(S_ij - m_i)          (natural log)

Backward (the pages only say that score blocks are recomputed from Q, K, V;
the gradient formulas are calculus on the definition above, with dO the
incoming gradient of O and LSE treated as a non-differentiable side output):

    dV = P^T dO
    dP = dO V^T
    D_i = sum_k dO_ik O_ik            (= sum_j P_ij dP_ij)
    dS = P * (dP - D)                 (elementwise, D broadcast over j)
    dQ = scale * dS K
    dK = scale * dS^T Q

Readings where the pages are silent (all recorded in the design notes):
* one LSE per row in natural-log units replaces the "two numbers per row"
  (running max and running sum) because P = exp(S - LSE) recovers both;
* causal masking is top-left aligned (key j visible to query i iff j <= i),
  the only reading with equal query and key lengths;
* inputs are the exact values the GPU sees (bf16 or fp32 widened to fp64) and
  ``scale`` is the fp32 value the GPU receives, widened;
* grouped-query attention ("Flash Attention" (karlkratz.de), "Grouped Query
  Attention") groups consecutive query heads: head h reads K/V head
  h // (H / Hkv);
* a sliding window ("Flash Attention" (karlkratz.de), "Sliding Window
  Attention") is a (left, right) pair: key j is visible to query i when
  i - left <= j <= i + right; the page's window of 4096 tokens is
  (4095, 0), the position and the 4095 before it.
* a block-sparse mask ("Flash Attention" (Ultralytics glossary), "Flash
  Attention и смежные понятия") is a 0/1 array over 128 x 128 blocks of the
  score matrix (one per query head, or one shared); a row whose blocks are all
  0 sees no key and gets O = 0, LSE = -inf.

* a paged KV cache ("Flash Attention" (Ultralytics glossary), "Flash Attention
  и смежные понятия", PagedAttention: the cache lives in fixed-size pages and
  the attention kernel reads keys and values from them) is a pool
  [num_pages, page_size, Hkv, d] plus a per-sequence page list: position j of
  sequence b is slot j % page_size of page block_table[b, j // page_size].  A
  decode step is one query per sequence attending to all seqlens[b] cached
  positions (none hidden); a sequence with no cached position gets O = 0,
  LSE = -inf.

``blocked_forward_head`` restates the pages' online-softmax algorithm (key
blocks streamed, running row max and sum, rescale when the max grows) and is
used only to pin the oracle: blocked and full results must agree.

Parity pins: every function here is pinned by ``tests/test_oracle.py``
(closed forms, invariants, finite differences, the pages' worked example).
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "hidden_keys",
    "scores_head",
    "probs_head",
    "forward_head",
    "forward_rows_head",
    "backward_head",
    "blocked_forward_head",
    "forward",
    "backward",
    "kv_head",
    "paged_rows",
    "decode_paged",
]


def _f64(x) -> np.ndarray:
    a = np.asarray(x)
    return a.astype(np.float64, copy=False)


def hidden_keys(rows, nk: int, causal: bool, window=None, block_mask=None, block: int = 128) -> np.ndarray:
    """Boolean [len(rows), nk] mask: True where key j is hidden from query row i.

    Query row i sits at sequence position i (top-left alignment).
    * causal: key j is hidden when j > i.
    * window = (left, right): key j is visible only when i - left <= j <= i + right;
      None on a side leaves that side unbounded.  "Flash Attention"
      (karlkratz.de), section "Sliding Window Attention": each position attends
      to a fixed neighbourhood; the page's 4096-token window is read as
      (left, right) = (4095, 0): the position itself and the 4095 before it.
    * block_mask: a [ceil(Nq / block), ceil(nk / block)] array; key j is hidden
      from row i when block_mask[i // block, j // block] is 0.  "Flash
      Attention" (Ultralytics glossary), "Flash Attention и смежные понятия":
      sparse attention scores only chosen query/key pairs, and the block-sparse
      form skips the empty blocks.
    The conditions combine: a key is visible only when every given one allows it.
    """
    rows = np.asarray(rows, dtype=np.int64)[:, None]
    cols = np.arange(nk)[None, :]
    hidden = np.zeros((rows.shape[0], nk), dtype=bool)
    if causal:
        hidden |= cols > rows
    if window is not None:
        left, right = window
        if right is not None:
            hidden |= cols > rows + right
        if left is not None:
            hidden |= cols < rows - left
    if block_mask is not None:
        bm = np.asarray(block_mask) != 0
        hidden |= ~bm[rows // block, cols // block]
    return hidden


def scores_head(q, k, scale: float, causal: bool, window=None, block_mask=None) -> np.ndarray:
    """S = scale * Q K^T for one (batch, head), with the mask applied.

    q: [Nq, d], k: [Nk, d].  Masked entries are -inf (see ``hidden_keys`` for
    the causal and sliding-window masks).  Standard attention as defined in
    "Flash Attention" (Ultralytics glossary), "Flash Attention и смежные
    понятия" (the same operation with the full score matrix written out).
    """
    q = _f64(q)
    k = _f64(k)
    s = float(scale) * (q @ k.T)
    if causal or window is not None or block_mask is not None:
        hidden = hidden_keys(np.arange(s.shape[0]), s.shape[1], causal, window, block_mask)
        s = np.where(hidden, -np.inf, s)
    return s


def probs_head(s: np.ndarray):
    """Row softmax of a score matrix.  Returns (P, LSE) with LSE natural-log.

    A row whose entries are all -inf (no visible key) gets P = 0 and
    LSE = -inf; with equal query and key lengths causal masking never
    produces one.
    """
    m = np.max(s, axis=1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    l = np.sum(e, axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
        lse = np.where(l[:, 0] > 0, m_safe[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)), -np.inf)
    return p, lse


def forward_head(q, k, v, scale: float, causal: bool, window=None, block_mask=None):
    """O = softmax(scale Q K^T + mask) V and LSE for one (batch, head).

    q, k, v: [N, d].  Returns O [N, d] float64 and LSE [N] float64.
    Definition of the exact result the tiled kernel must reproduce:
    "Flash Attention" (karlkratz.de), "Speicherbedarf und Laufzeitverhalten"
    (same result, not an approximation).
    """
    s = scores_head(q, k, scale, causal, window, block_mask)
    p, lse = probs_head(s)
    return p @ _f64(v), lse


def forward_rows_head(q, k, v, rows, scale: float, causal: bool, window=None, block_mask=None):
    """Forward restricted to the query rows ``rows`` of one (batch, head).

    A row of O and its LSE depend only on that query row and all of K and V,
    so this is the definition evaluated on a subset of rows (used to check
    large problems on sampled rows).
    """
    rows = np.asarray(rows, dtype=np.int64)
    q = _f64(q)
    k = _f64(k)
    s = float(scale) * (q[rows] @ k.T)
    if causal or window is not None or block_mask is not None:
        s = np.where(hidden_keys(rows, k.shape[0], causal, window, block_mask), -np.inf, s)
    p, lse = probs_head(s)
    return p @ _f64(v), lse


def backward_head(q, k, v, do, scale: float, causal: bool, window=None, block_mask=None):
    """Gradients (dQ, dK, dV) of O = attention(Q, K, V) given dO, one head.

    Recomputes S and P from Q, K and V ("Flash Attention" (karlkratz.de),
    "Recomputation beim Rückwärtsdurchlauf": the backward recomputes the
    attention values instead of storing them).  Also returns D = rowsum(dO*O).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    s = scores_head(q, k, scale, causal, window, block_mask)
    p, _ = probs_head(s)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    dvec = np.sum(do * o, axis=1)
    ds = p * (dp - dvec[:, None])
    dq = float(scale) * (ds @ k)
    dk = float(scale) * (ds.T @ q)
    return dq, dk, dv, dvec


def blocked_forward_head(q, k, v, scale: float, causal: bool, block: int,
                         tau: float = 0.0, dtype=np.float64):
    """Online-softmax forward over key blocks, as the pages describe it.

    Follows "Flash Attention" (Ultralytics glossary), "Принцип работы Flash
    Attention": all query rows are held at once, key/value blocks stream past;
    for each block the scores are formed, the running row maximum and running
    row sum are updated, the partial output is rescaled when the maximum
    grows, and the block's weighted values are added; finally the output is
    divided by the running sum.  "Flash Attention" (karlkratz.de), "Tiling"
    describes the same per-row pair (maximum, sum) and correction factor.

    ``tau`` > 0 is the lazy variant: the reference maximum is only moved when
    the new block maximum exceeds it by more than ``tau`` (natural-log units);
    numerator and denominator share the same reference, so the result is the
    same.  ``dtype`` selects the working precision (float64 for pins of the
    exact result, float32 to reproduce the pages' fp32 demonstration).
    Returns (O, LSE).
    """
    q = np.asarray(q, dtype=dtype)
    k = np.asarray(k, dtype=dtype)
    v = np.asarray(v, dtype=dtype)
    n, d = q.shape
    nk = k.shape[0]
    sc = dtype(scale)
    run_max = np.full((n, 1), -np.inf, dtype=dtype)
    run_sum = np.zeros((n, 1), dtype=dtype)
    acc = np.zeros((n, v.shape[1]), dtype=dtype)
    rows = np.arange(n)[:, None]
    for start in range(0, nk, block):
        stop = min(start + block, nk)
        s = (q @ k[start:stop].T) * sc
        if causal:
            cols = np.arange(start, stop)[None, :]
            s = np.where(cols > rows, dtype(-np.inf), s)
        blk_max = np.max(s, axis=1, keepdims=True)
        cand = np.maximum(run_max, blk_max)
        move = cand > run_max + dtype(tau) if tau > 0 else cand > run_max
        new_max = np.where(move | ~np.isfinite(run_max), cand, run_max)
        base = np.where(np.isfinite(new_max), new_max, dtype(0))
        with np.errstate(invalid="ignore"):
            corr = np.where(np.isfinite(run_max), np.exp(run_max - base), dtype(0))
        e = np.exp(s - base)
        run_sum = run_sum * corr + np.sum(e, axis=1, keepdims=True)
        acc = acc * corr + e @ v[start:stop]
        run_max = new_max
    with np.errstate(divide="ignore", invalid="ignore"):
        out = np.where(run_sum > 0, acc / np.where(run_sum > 0, run_sum, 1), 0)
        lse = np.where(run_sum[:, 0] > 0,
                       np.where(np.isfinite(run_max[:, 0]), run_max[:, 0], 0)
                       + np.log(np.where(run_sum[:, 0] > 0, run_sum[:, 0], 1)), -np.inf)
    return out.astype(dtype), lse.astype(dtype)


def kv_head(h: int, n_heads: int, n_kv_heads: int) -> int:
    """K/V head read by query head ``h`` under grouped-query attention.

    "Flash Attention" (karlkratz.de), section "Grouped Query Attention":
    several query heads share one K/V group (64 query heads on 8 K/V heads in
    the page's example).  The page does not fix which heads share; the reading
    taken is consecutive groups, query head h -> K/V head h // (H / Hkv), so
    Hkv = H is ordinary multi-head attention and Hkv = 1 multi-query attention.
    """
    if n_kv_heads < 1 or n_heads % n_kv_heads:
        raise ValueError("the K/V head count must divide the query head count")
    return h // (n_heads // n_kv_heads)


def _head_mask(block_mask, h):
    if block_mask is None:
        return None
    bm = np.asarray(block_mask)
    return bm[h] if bm.ndim == 3 else bm


def forward(Q, K, V, scale: float, causal: bool, heads=None, window=None, block_mask=None):
    """Batched forward: Q [B, N, H, d]; K, V [B, N, Hkv, d] (numpy or CPU torch).

    Returns O [B, N, H, d] and LSE [B, H, N] in float64.  ``heads`` restricts
    the work to a list of (b, h) query-head pairs; other entries are left as
    NaN.  With Hkv < H each query head attends with K/V head ``kv_head(h)``.
    """
    Q, K, V = (_f64(_to_numpy(t)) for t in (Q, K, V))
    b_, n_, h_, d_ = Q.shape
    hkv = K.shape[2]
    O = np.full((b_, n_, h_, V.shape[3]), np.nan)
    LSE = np.full((b_, h_, n_), np.nan)
    for (b, h) in (heads if heads is not None else _all_heads(b_, h_)):
        g = kv_head(h, h_, hkv)
        o, lse = forward_head(Q[b, :, h], K[b, :, g], V[b, :, g], scale, causal, window, _head_mask(block_mask, h))
        O[b, :, h] = o
        LSE[b, h] = lse
    return O, LSE


def backward(Q, K, V, dO, scale: float, causal: bool, heads=None, window=None, block_mask=None):
    """Batched backward.  Returns dQ [B, N, H, d], dK and dV [B, N, Hkv, d] (float64).

    A K/V head shared by a group of query heads enters each of their
    attentions, so its gradient is the sum of the per-query-head gradients
    (chain rule).  With ``heads`` given, dK and dV sum over the listed query
    heads only (entries no listed head touches stay NaN).
    """
    Q, K, V, dO = (_f64(_to_numpy(t)) for t in (Q, K, V, dO))
    shape = Q.shape
    hkv = K.shape[2]
    dQ = np.full(shape, np.nan)
    dK = np.full(K.shape, np.nan)
    dV = np.full(V.shape, np.nan)
    touched = set()
    for (b, h) in (heads if heads is not None else _all_heads(shape[0], shape[2])):
        g = kv_head(h, shape[2], hkv)
        dq, dk, dv, _ = backward_head(Q[b, :, h], K[b, :, g], V[b, :, g], dO[b, :, h], scale, causal, window,
                                      _head_mask(block_mask, h))
        dQ[b, :, h] = dq
        if (b, g) not in touched:
            touched.add((b, g))
            dK[b, :, g] = 0.0
            dV[b, :, g] = 0.0
        dK[b, :, g] += dk
        dV[b, :, g] += dv
    return dQ, dK, dV


def _all_heads(nb, nh):
    return [(b, h) for b in range(nb) for h in range(nh)]


def _to_numpy(t):
    if hasattr(t, "detach"):
        t = t.detach()
        if hasattr(t, "dtype") and str(t.dtype) == "torch.bfloat16":
            t = t.float()
        return t.cpu().numpy()
    return np.asarray(t)


def paged_rows(cache, table_row, length: int) -> np.ndarray:
    """The first ``length`` cached rows of one sequence, gathered from a page pool.

    cache: [num_pages, page_size, ...] (numpy or CPU torch); table_row: the
    sequence's page list.  Position j sits in slot j % page_size of page
    table_row[j // page_size] ("Flash Attention" (Ultralytics glossary), "Flash
    Attention и смежные понятия", PagedAttention: keys and values are read from
    fixed-size pages).  Returns [length, ...] float64.
    """
    cache = _f64(_to_numpy(cache))
    table_row = np.asarray(_to_numpy(table_row), dtype=np.int64)
    page_size = cache.shape[1]
    out = np.empty((length,) + cache.shape[2:])
    for j in range(length):
        out[j] = cache[table_row[j // page_size], j % page_size]
    return out


def decode_paged(Q, K_cache, V_cache, block_table, seqlens, scale: float):
    """One decode step of attention over a paged KV cache.

    Q: [B, H, d] (one new query per sequence); K_cache, V_cache:
    [num_pages, page_size, Hkv, d]; block_table: [B, max_pages] page indices;
    seqlens: [B] cached positions per sequence.  Query head h of sequence b
    attends, with K/V head ``kv_head(h)``, to the seqlens[b] rows that
    ``paged_rows`` gathers: the plain definition (``forward_rows_head``, no
    mask) on the gathered rows.  Returns O [B, H, d] and LSE [B, H] (float64);
    a sequence with no cached position gets O = 0 and LSE = -inf.
    """
    Q = _f64(_to_numpy(Q))
    K_cache, V_cache = (_f64(_to_numpy(t)) for t in (K_cache, V_cache))
    table = np.asarray(_to_numpy(block_table), dtype=np.int64)
    lens = np.asarray(_to_numpy(seqlens), dtype=np.int64)
    nb, nh, d = Q.shape
    hkv = K_cache.shape[2]
    O = np.zeros((nb, nh, V_cache.shape[3]))
    LSE = np.full((nb, nh), -np.inf)
    for b in range(nb):
        n = int(lens[b])
        if n == 0:
            continue
        k_rows = paged_rows(K_cache, table[b], n)  # [n, Hkv, d]
        v_rows = paged_rows(V_cache, table[b], n)
        for h in range(nh):
            g = kv_head(h, nh, hkv)
            o, lse = forward_rows_head(Q[b, h][None, :], k_rows[:, g], v_rows[:, g], [0], scale, False)
            O[b, h] = o[0]
            LSE[b, h] = lse[0]
    return O, LSE
