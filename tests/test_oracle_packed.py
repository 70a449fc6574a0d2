"""Pins for the packed (variable-length) oracle.

The oracle slices the packed tensors into sequences and applies the padded
definition to each slice.  These tests check it against a formulation that
slices nothing: attention over the whole packed stream with a block-diagonal
"same sequence" mask, written with PyTorch's float64 softmax, logsumexp and
autograd.  Further pins: equal lengths reduce to the padded oracle, empty and
one-token sequences, dropout masks placed block-diagonally, and planted
mistakes (a packed oracle that lets sequences see each other, or that
measures ALiBi / window distances from the start of the pack) that the
segment pin must catch.
"""

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import packed as op
from oracle import philox

RNG = np.random.default_rng(777)


def pack(lengths, H, d, scale=1.0):
    total = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    q, k, v, do = (RNG.standard_normal((total, H, d)) * scale for _ in range(4))
    return q, k, v, do, cu


def segment_attention(q, k, v, cu, scale, causal=False, wl=-1, wr=-1, slopes=None,
                      keep=None, keep_scale=1.0):
    """Attention over the whole packed stream (torch float64, autograd-able):
    key r is visible to query t iff both lie in the same sequence and the
    window/causal conditions hold for their distance t - r."""
    total = q.shape[0]
    lengths = np.diff(cu)
    seg = torch.repeat_interleave(torch.arange(len(lengths)), torch.as_tensor(lengths))
    t = torch.arange(total)
    same = seg[:, None] == seg[None, :]
    rel = t[None, :] - t[:, None]                      # r - t
    ok = same.clone()
    if causal:
        ok &= rel <= 0
    if wl >= 0:
        ok &= rel >= -wl
    if wr >= 0:
        ok &= rel <= wr
    s = scale * torch.einsum("thd,rhd->htr", q, k)
    if slopes is not None:
        s = s - torch.as_tensor(slopes, dtype=torch.float64)[:, None, None] * rel.abs()
    s = s.masked_fill(~ok, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)                   # [H, total]
    p = torch.softmax(s, dim=-1)
    if keep is not None:
        p = p * torch.as_tensor(keep) * keep_scale
    o = torch.einsum("htr,rhd->thd", p, v)
    return o, lse


def seg_fwd_bwd(q, k, v, do, cu, scale, **kw):
    qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o, lse = segment_attention(qt, kt, vt, cu, scale, **kw)
    (o * torch.tensor(do)).sum().backward()
    return (o.detach().numpy(), lse.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(),
            vt.grad.numpy())


CASES = [
    dict(lengths=[5, 1, 9, 0, 7], causal=False),
    dict(lengths=[5, 1, 9, 0, 7], causal=True),
    dict(lengths=[12, 3, 8], causal=True, wl=4, wr=0),
    dict(lengths=[12, 3, 8], wl=2, wr=3),
    dict(lengths=[10, 6, 11], causal=True, alibi=True),
    dict(lengths=[0, 0, 4, 0], causal=False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: str(c))
def test_packed_matches_segment_mask(case):
    H, d, scale = 3, 8, 0.4
    q, k, v, do, cu = pack(case["lengths"], H, d)
    slopes = np.array([0.5, 0.25, 0.125]) if case.get("alibi") else None
    kw = dict(causal=case.get("causal", False), wl=case.get("wl", -1), wr=case.get("wr", -1),
              slopes=slopes)
    o_s, lse_s, dq_s, dk_s, dv_s = seg_fwd_bwd(q, k, v, do, cu, scale, **kw)
    okw = dict(causal=kw["causal"], window_left=kw["wl"], window_right=kw["wr"],
               alibi_slopes=slopes)
    o, lse = op.packed_forward(q, k, v, cu, scale, **okw)
    assert np.allclose(o, o_s, atol=1e-12)
    assert np.allclose(lse, lse_s, atol=1e-12)
    dq, dk, dv, dvec = op.packed_backward(q, k, v, do, cu, scale, **okw)
    assert np.allclose(dq, dq_s, atol=1e-12)
    assert np.allclose(dk, dk_s, atol=1e-12)
    assert np.allclose(dv, dv_s, atol=1e-12)
    assert np.allclose(dvec, np.einsum("thd,thd->ht", do, o), atol=1e-12)


def test_equal_lengths_reduce_to_padded():
    B, N, H, d, scale = 3, 9, 2, 8, 0.3
    q, k, v, do, cu = pack([N] * B, H, d)
    o, lse = op.packed_forward(q, k, v, cu, scale, causal=True)
    o_p, lse_p = oa.attention_forward(q.reshape(B, N, H, d), k.reshape(B, N, H, d),
                                      v.reshape(B, N, H, d), scale, causal=True)
    assert np.allclose(o, o_p.reshape(B * N, H, d), atol=1e-14)
    assert np.allclose(lse, lse_p.transpose(1, 0, 2).reshape(H, B * N), atol=1e-14)
    dq, dk, dv, _ = op.packed_backward(q, k, v, do, cu, scale, causal=True)
    r = oa.attention_backward(*(x.reshape(B, N, H, d) for x in (q, k, v, do)), scale,
                              causal=True)
    for got, ref in zip((dq, dk, dv), r[:3]):
        assert np.allclose(got, ref.reshape(B * N, H, d), atol=1e-14)


def test_one_token_sequences_copy_v():
    # a sequence of one token sees only itself: O = v, LSE = scale <q, k>
    q, k, v, _, cu = pack([1, 1, 1], 2, 4)
    o, lse = op.packed_forward(q, k, v, cu, 0.5)
    assert np.allclose(o, v, atol=1e-15)
    assert np.allclose(lse, 0.5 * np.einsum("thd,thd->ht", q, k), atol=1e-14)


def test_dropout_is_block_diagonal_per_sequence():
    lengths, H, d, scale, p, seed = [6, 0, 9, 4], 2, 8, 0.35, 0.3, 99
    q, k, v, do, cu = pack(lengths, H, d)
    ks = philox.keep_scale(p)

    def keep(b, h, n):
        return philox.keep_mask(b, h, np.arange(n), n, p, seed)

    total = sum(lengths)
    full = np.zeros((H, total, total))
    for b, (s, e) in enumerate(op.spans(cu)):
        for h in range(H):
            full[h, s:e, s:e] = keep(b, h, e - s)
    o_s, lse_s, dq_s, dk_s, dv_s = seg_fwd_bwd(q, k, v, do, cu, scale, causal=True,
                                               keep=full, keep_scale=ks)
    o, lse = op.packed_forward(q, k, v, cu, scale, causal=True, keep=keep, keep_scale=ks)
    assert np.allclose(o, o_s, atol=1e-12) and np.allclose(lse, lse_s, atol=1e-12)
    dq, dk, dv, _ = op.packed_backward(q, k, v, do, cu, scale, causal=True, keep=keep,
                                       keep_scale=ks)
    for got, ref in ((dq, dq_s), (dk, dk_s), (dv, dv_s)):
        assert np.allclose(got, ref, atol=1e-12)


def test_spans_rejects_malformed_offsets():
    assert op.spans([0, 3, 3, 7]) == [(0, 3), (3, 3), (3, 7)]
    for bad in ([1, 3], [0, 4, 2], []):
        with pytest.raises(ValueError):
            op.spans(bad)


def test_planted_mistakes_fail_the_segment_pin():
    lengths, H, d, scale = [7, 5, 8], 2, 8, 0.4
    q, k, v, _, cu = pack(lengths, H, d)
    slopes = np.array([0.5, 0.25])
    o_s, _ = segment_attention(*(torch.tensor(x) for x in (q, k, v)), cu, scale, causal=True,
                               wl=3, slopes=slopes)
    o_s = o_s.numpy()
    # (1) sequences see each other: the whole pack as one causal sequence
    o1 = np.stack([oa.head_forward(q[:, h], k[:, h], v[:, h], scale, True, 3, -1,
                                   slopes[h])[0] for h in range(H)], axis=1)
    assert not np.allclose(o1, o_s, atol=1e-6)
    # (2) positions measured from the start of the pack: query rows of a later
    # sequence evaluated with global row indices against its own keys
    o2 = np.zeros_like(o_s)
    for s, e in op.spans(cu):
        for h in range(H):
            rows = np.arange(s, e)
            kk = np.zeros((e, d))
            vv = np.zeros((e, d))
            kk[s:e], vv[s:e] = k[s:e, h], v[s:e, h]
            # keys before s are zero vectors standing in for "not this sequence"
            o2[s:e, h] = oa.head_forward(q[s:e, h], kk, vv, scale, True, 3, -1, slopes[h],
                                         rows=rows)[0]
    assert not np.allclose(o2, o_s, atol=1e-6)
    # the correct oracle passes the same pin
    o, _ = op.packed_forward(q, k, v, cu, scale, causal=True, window_left=3,
                             alibi_slopes=slopes)
    assert np.allclose(o, o_s, atol=1e-12)
