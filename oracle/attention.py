"""Plain fp64 definition of exact softmax attention and its gradient.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline legs of ``bench.py``.  The CUDA library never calls
into this module and this module shares no code with it.

What is computed, and where the pages fix it
--------------------------------------------
* The result is the ordinary attention of a Transformer, unchanged: the
  FlashAttention explainer "AI基础 | Flash Attention" (yeyulingfeng.com)
  says in its opening section that Flash Attention computes exactly the
  same attention and the same result, only organised differently on the
  GPU; the FlashAttention-2 abstract (arXiv 2307.08691) says "without
  approximation".  So the oracle is the textbook definition, written out:
  materialise the N x N scores, softmax each row in two passes (row max,
  then exponentials of the differences divided by their sum, as the
  explainer's "Online softmax" section describes standard softmax), and
  multiply by V.
* The call's options come from the "FlashAttention v2" article (wmrh.cn),
  §5.1 (API): ``softmax_scale`` (None -> 1/sqrt(d), the plain reading),
  ``causal``, ``window_size=(left, right)`` (-1 = unbounded) and
  ``alibi_slopes`` (a linear positional bias per head).
* The backward pass recomputes the probabilities from the inputs (the
  explainer's "Backward pass" section: only per-row statistics are kept
  from the forward pass).  The gradients are the textbook softmax/matmul
  gradients; the pages print no formula, so these are the plain reading:
      dV = P^T dO,   dP = dO V^T,   D_i = sum_c dO_ic O_ic,
      dS = P * (dP - D 1^T),   dQ = scale dS K,   dK = scale dS^T Q.
* The per-row statistic returned by the forward pass is the natural-log
  log-sum-exp, LSE_i = M_i + ln(l_i) with M_i the row max of the scaled,
  biased scores and l_i = sum_j exp(s_ij - M_i) (the "running max and
  running sum" of the explainer's "Backward pass" section, folded into one
  number).

Readings taken where the pages are silent (each repeated where it applies):
* window bounds are inclusive: key j is visible to query i iff
  i - left <= j <= i + right, a negative bound meaning "unbounded";
* ``causal`` additionally requires j <= i;
* ALiBi adds -slope_h * |i - j| to the scaled score (for causal use i >= j,
  so this is -slope_h * (i - j));
* a row with no visible key (unreachable with the shipped masks, since the
  diagonal is always visible) has O = 0, LSE = -inf and zero gradients.

Block-sparse masks ("FlashAttention v2" article, §6, future work: block-
sparse attention; the pages give no formula, so the plain reading is
taken): a boolean block mask M of shape [ceil(N / block), ceil(N / block)]
per head hides key j from query i unless M[i // block, j // block] is true,
on top of the causal and window masks.  The library's block is 128.

Dropout (the call's ``dropout_p``; the pages give no formula, so the plain
reading of attention dropout is taken): after the softmax, each probability
is kept or zeroed by a given boolean mask and kept ones are multiplied by a
given scale (1 / keep probability); O = (P o keep * scale) V, while LSE stays
the log-sum-exp of the un-dropped scores.  The mask is an INPUT here (it is
drawn by oracle/philox.py), so these functions hold no random-number code.
In the backward pass the same mask multiplies dO V^T, and D = rowsum(dO o O)
with the dropped O is still sum_j P_ij dP_ij.

Layouts: q, k, v, o, do, dq, dk, dv are [B, N, H, d]; lse and D are
[B, H, N].  All arithmetic is float64; callers pass the exact values the GPU
receives (e.g. bf16 inputs widened to float64).
"""

from __future__ import annotations

import math

import numpy as np

# Largest score matrix (in float64 elements) materialised at once.  Query rows
# of the forward pass are independent, so a long head is processed in chunks
# of rows; the backward's sums over query rows (dK, dV) are then accumulated
# chunk by chunk, a reassociation of the same fp64 sum.
_MAX_SCORE_ELEMS = 1 << 26


def allowed_mask(rows: np.ndarray, n_keys: int, causal: bool,
                 window_left: int, window_right: int) -> np.ndarray:
    """Boolean [len(rows), n_keys]: True where query ``i`` may see key ``j``.

    "FlashAttention v2" article (wmrh.cn), §5.1: ``causal`` and the local
    window ``window_size=(left, right)``, -1 meaning no bound.  Inclusive
    bounds are the reading taken.
    """
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(n_keys, dtype=np.int64)[None, :]
    ok = np.ones((i.shape[0], n_keys), dtype=bool)
    if causal:
        ok &= j <= i
    if window_left >= 0:
        ok &= j >= i - window_left
    if window_right >= 0:
        ok &= j <= i + window_right
    return ok


def block_mask_elements(block_mask, rows, n_keys: int, block: int) -> np.ndarray:
    """Boolean [len(rows), n_keys]: True where block (i // block, j // block)
    of the block mask is set."""
    bm = np.asarray(block_mask, dtype=bool)
    i = np.asarray(rows, dtype=np.int64) // block
    j = np.arange(n_keys, dtype=np.int64) // block
    return bm[i[:, None], j[None, :]]


def alibi_bias(rows: np.ndarray, n_keys: int, slope: float) -> np.ndarray:
    """ALiBi bias -slope * |i - j| ("FlashAttention v2" article, §5.1,
    ``alibi_slopes``; sign and |i-j| form are the reading taken)."""
    i = np.asarray(rows, dtype=np.float64)[:, None]
    j = np.arange(n_keys, dtype=np.float64)[None, :]
    return -float(slope) * np.abs(i - j)


def head_scores(q_rows: np.ndarray, k: np.ndarray, rows: np.ndarray,
                scale: float, causal: bool, window_left: int,
                window_right: int, slope: float | None,
                block_mask=None, block: int = 128) -> np.ndarray:
    """s_ij = scale * <q_i, k_j> + bias_ij, -inf where the mask hides j."""
    s = scale * (q_rows @ k.T)
    if slope is not None:
        s = s + alibi_bias(rows, k.shape[0], slope)
    ok = allowed_mask(rows, k.shape[0], causal, window_left, window_right)
    if block_mask is not None:
        ok &= block_mask_elements(block_mask, rows, k.shape[0], block)
    return np.where(ok, s, -np.inf)


def _softmax_rows(s: np.ndarray):
    """Two-pass softmax of each row: max, then exp(s - max) / sum.

    Returns (P, M, l).  Rows that are entirely -inf give P = 0, M = -inf,
    l = 0.
    """
    m = s.max(axis=1)
    dead = ~np.isfinite(m)
    m_safe = np.where(dead, 0.0, m)
    e = np.exp(s - m_safe[:, None])          # exp(-inf) = 0 for hidden keys
    l = e.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        p = np.where(dead[:, None], 0.0, e / np.where(dead, 1.0, l)[:, None])
    return p, m, l


def head_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                 causal: bool = False, window_left: int = -1,
                 window_right: int = -1, slope: float | None = None,
                 rows: np.ndarray | None = None, keep=None,
                 keep_scale: float = 1.0, block_mask=None, block: int = 128):
    """One head: q [Nq_rows, d] (the rows listed in ``rows``), k, v [N, d].

    ``keep`` (optional): boolean [len(rows), N] dropout mask, applied to P
    with ``keep_scale``.  ``block_mask`` (optional): boolean block mask of
    this head (see the module docstring).  Returns (O [rows, d], LSE [rows])
    with LSE = M + ln(l) of the un-dropped scores.
    """
    n = k.shape[0]
    if rows is None:
        rows = np.arange(q.shape[0])
    rows = np.asarray(rows, dtype=np.int64)
    o = np.zeros((rows.shape[0], v.shape[1]), dtype=np.float64)
    lse = np.full(rows.shape[0], -np.inf, dtype=np.float64)
    chunk = max(1, _MAX_SCORE_ELEMS // max(n, 1))
    for r0 in range(0, rows.shape[0], chunk):
        rr = rows[r0:r0 + chunk]
        s = head_scores(q[r0:r0 + chunk], k, rr, scale, causal, window_left,
                        window_right, slope, block_mask, block)
        p, m, l = _softmax_rows(s)
        if keep is not None:
            p = p * (keep[r0:r0 + chunk] * keep_scale)
        o[r0:r0 + chunk] = p @ v
        live = np.isfinite(m)
        lse[r0:r0 + chunk] = np.where(live, m + np.log(np.where(live, l, 1.0)),
                                      -np.inf)
    return o, lse


def head_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                  do: np.ndarray, scale: float, causal: bool = False,
                  window_left: int = -1, window_right: int = -1,
                  slope: float | None = None, keep=None,
                  keep_scale: float = 1.0, block_mask=None, block: int = 128):
    """Textbook gradients for one head (q, k, v, do are [N, d]).

    The probabilities are recomputed from the inputs, as in the explainer's
    "Backward pass" section.  ``keep``: optional [N, N] dropout mask (see the
    module docstring).  Returns (dq, dk, dv, D) with D_i = sum_c dO_ic O_ic.
    """
    n, d = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dvec = np.zeros(n, dtype=np.float64)
    chunk = max(1, _MAX_SCORE_ELEMS // max(n, 1))
    for r0 in range(0, n, chunk):
        rr = np.arange(r0, min(n, r0 + chunk))
        s = head_scores(q[rr], k, rr, scale, causal, window_left,
                        window_right, slope, block_mask, block)
        p, _, _ = _softmax_rows(s)
        mk = 1.0 if keep is None else keep[rr] * keep_scale
        pd = p * mk                            # dropped probabilities
        o = pd @ v
        do_r = do[rr]
        dv += pd.T @ do_r                      # dV = (P o keep)^T dO
        dp = (do_r @ v.T) * mk                 # dP = (dO V^T) o keep
        d_r = np.sum(do_r * o, axis=1)         # D = rowsum(dO o O)
        ds = p * (dp - d_r[:, None])           # dS = P o (dP - D)
        dq[rr] = scale * (ds @ k)              # dQ = scale dS K
        dk += scale * (ds.T @ q[rr])           # dK = scale dS^T Q
        dvec[rr] = d_r
    return dq, dk, dv, dvec


def _slope(alibi_slopes, h):
    return None if alibi_slopes is None else float(alibi_slopes[h])


def attention_forward(q, k, v, scale: float, causal: bool = False,
                      window_left: int = -1, window_right: int = -1,
                      alibi_slopes=None, heads=None, block_mask=None,
                      block: int = 128):
    """O [B,N,H,d] and LSE [B,H,N] for every (b, h), or only for the
    (b, h) pairs listed in ``heads`` (other entries are left NaN).
    ``block_mask``: optional boolean [B, H, nq_blocks, nk_blocks]."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    b_, n, h_, d = q.shape
    o = np.full((b_, n, h_, v.shape[3]), np.nan)
    lse = np.full((b_, h_, n), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(b_)
                                             for h in range(h_)]
    for b, h in pairs:
        o[b, :, h], lse[b, h] = head_forward(
            q[b, :, h], k[b, :, h], v[b, :, h], scale, causal, window_left,
            window_right, _slope(alibi_slopes, h),
            block_mask=None if block_mask is None else block_mask[b][h],
            block=block)
    return o, lse


def attention_forward_rows(q, k, v, b: int, h: int, rows, scale: float,
                           causal: bool = False, window_left: int = -1,
                           window_right: int = -1, alibi_slopes=None):
    """O and LSE for selected query rows of head (b, h); rows of the forward
    pass are independent, so this equals the matching rows of the full
    result."""
    rows = np.asarray(rows, dtype=np.int64)
    qb = np.asarray(q[b, rows, h], dtype=np.float64)
    return head_forward(qb, np.asarray(k[b, :, h], dtype=np.float64),
                        np.asarray(v[b, :, h], dtype=np.float64), scale,
                        causal, window_left, window_right,
                        _slope(alibi_slopes, h), rows=rows)


def attention_backward(q, k, v, do, scale: float, causal: bool = False,
                       window_left: int = -1, window_right: int = -1,
                       alibi_slopes=None, heads=None, block_mask=None,
                       block: int = 128):
    """dq, dk, dv [B,N,H,d] and D [B,H,N] (all heads, or those in ``heads``;
    other entries are left NaN)."""
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    b_, n, h_, d = q.shape
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    dvec = np.full((b_, h_, n), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(b_)
                                             for h in range(h_)]
    for b, h in pairs:
        dq[b, :, h], dk[b, :, h], dv[b, :, h], dvec[b, h] = head_backward(
            q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale, causal,
            window_left, window_right, _slope(alibi_slopes, h),
            block_mask=None if block_mask is None else block_mask[b][h],
            block=block)
    return dq, dk, dv, dvec


def bwd_preprocess(o, do):
    """D[b, h, i] = sum_c dO[b, i, h, c] * O[b, i, h, c] in float64."""
    o = np.asarray(o, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    return np.einsum("bnhd,bnhd->bhn", do, o)


def default_scale(d: int) -> float:
    """``softmax_scale=None`` read as 1/sqrt(d) ("FlashAttention v2"
    article, §5.1 lists the argument; the value is the plain reading)."""
    return 1.0 / math.sqrt(d)
