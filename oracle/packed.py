"""Packed variable-length batches: each sequence attended to on its own.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): used by ``tests/``
and ``bench.py``'s CPU legs; it shares no code with the CUDA library.

"Dynamic sequence support" is named as future work in §6 of the
"FlashAttention v2" article (wmrh.cn); the pages give no layout or formula,
so the plain reading is taken:

* B sequences of lengths L_0 .. L_{B-1} are stored back to back, with no
  padding, in tensors of ``total = sum L_b`` rows: q, k, v, o, do, dq, dk,
  dv are [total, H, d], and sequence b owns rows
  [cu_seqlens[b], cu_seqlens[b + 1]) with cu_seqlens[0] = 0.
* Sequence b is attended to exactly as if it were the only sequence of a
  padded batch: its queries see only its own keys, and the causal and
  window masks and the ALiBi distance |i - j| use positions 0 .. L_b - 1
  inside the sequence.  So the result is the padded definition of
  ``oracle/attention.py`` applied to each slice.
* Row statistics (LSE, D) are [H, total].
* Dropout: the keep mask of (sequence b, head h) is an INPUT, supplied by
  ``keep(b, h, n)`` -> bool [n, n] (the tests draw it with oracle/philox.py
  at batch index b, which is what a padded call of that sequence alone at
  batch index b would draw).

All arithmetic is float64.
"""

from __future__ import annotations

import numpy as np

from .attention import head_backward, head_forward


def spans(cu_seqlens):
    """[(start, end)] of every sequence, checking that cu_seqlens is a
    non-decreasing list of offsets starting at 0."""
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    if not cu or cu[0] != 0 or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must start at 0 and be non-decreasing")
    return list(zip(cu[:-1], cu[1:]))


def _slope(alibi_slopes, h):
    return None if alibi_slopes is None else float(alibi_slopes[h])


def packed_forward(q, k, v, cu_seqlens, scale: float, causal: bool = False,
                   window_left: int = -1, window_right: int = -1,
                   alibi_slopes=None, keep=None, keep_scale: float = 1.0):
    """O [total, H, d] and LSE [H, total] of a packed batch."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    total, n_heads, _ = q.shape
    o = np.zeros((total, n_heads, v.shape[2]))
    lse = np.full((n_heads, total), -np.inf)
    for b, (s, e) in enumerate(spans(cu_seqlens)):
        if e == s:
            continue
        for h in range(n_heads):
            mask = None if keep is None else keep(b, h, e - s)
            o[s:e, h], lse[h, s:e] = head_forward(
                q[s:e, h], k[s:e, h], v[s:e, h], scale, causal, window_left,
                window_right, _slope(alibi_slopes, h), keep=mask,
                keep_scale=keep_scale)
    return o, lse


def packed_backward(q, k, v, do, cu_seqlens, scale: float,
                    causal: bool = False, window_left: int = -1,
                    window_right: int = -1, alibi_slopes=None, keep=None,
                    keep_scale: float = 1.0):
    """dq, dk, dv [total, H, d] and D [H, total] of a packed batch."""
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    total, n_heads, _ = q.shape
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dvec = np.zeros((n_heads, total))
    for b, (s, e) in enumerate(spans(cu_seqlens)):
        if e == s:
            continue
        for h in range(n_heads):
            mask = None if keep is None else keep(b, h, e - s)
            dq[s:e, h], dk[s:e, h], dv[s:e, h], dvec[h, s:e] = head_backward(
                q[s:e, h], k[s:e, h], v[s:e, h], do[s:e, h], scale, causal,
                window_left, window_right, _slope(alibi_slopes, h),
                keep=mask, keep_scale=keep_scale)
    return dq, dk, dv, dvec
