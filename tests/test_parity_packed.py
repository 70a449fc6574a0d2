"""Packed (variable-length) batches: libfa2 against the fp64 oracle.

Every sequence of a packed call is compared with the oracle's attention of
that sequence alone (oracle/packed.py), element by element, forward and
backward.  The length mixes put sequence boundaries inside 128-row tiles,
use lengths 0 and 1, lengths just below and above tile and tile-pair
multiples, and several sequences shorter than one tile, so tiles that run
into the next sequence, empty units and row-wise output stores are all
exercised.  The packed result is also checked bit for bit against padded
calls of the same sequences one at a time, and a malformed cu_seqlens must
be reported through the device status word.
"""

import numpy as np
import pytest
import torch

from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W
from oracle import packed as op
from oracle import philox
from tests.helpers import assert_same_sum_any_order, check_fwd, check_grad, d_rounding_bounds, f64

pytestmark = pytest.mark.gpu

MIX = (300, 1, 0, 129, 513, 128, 256, 77, 640)

CASES = [
    W.packed("mix-d128", MIX, H=2, d=128, seed=71),
    W.packed("mix-d128-causal", MIX, H=2, d=128, causal=True, seed=72),
    W.packed("mix-d64", MIX, H=2, d=64, seed=73),
    W.packed("mix-d64-causal", MIX, H=2, d=64, causal=True, seed=74),
    W.packed("window", (700, 5, 390), H=2, d=128, causal=True, window_left=130,
             window_right=0, seed=75),
    W.packed("window-both", (600, 200), H=2, d=64, window_left=5, window_right=7, seed=76),
    W.packed("alibi", (520, 3, 260), H=3, d=128, causal=True, alibi=True, seed=77),
    W.packed("det", (384, 129, 1, 700), H=2, d=128, causal=True, deterministic=True, seed=78),
    W.packed("det-d64", (300, 513), H=2, d=64, deterministic=True, seed=79),
    W.packed("single", (1000,), H=2, d=128, seed=80),
    W.packed("fp32", (200, 1, 65), H=2, d=64, dtype=torch.float32, causal=True, seed=81,
             scale=1.0 / 8.0),
    W.packed("fp32-d128", (100, 37), H=1, d=128, dtype=torch.float32, seed=82),
]


def run(w, dropout_p=0.0, seed=0):
    q, k, v, do = W.make_inputs(w, "cuda")
    cu = w.cu_seqlens("cuda")
    slopes = w.alibi_slopes()
    sl = None if slopes is None else slopes.cuda()
    win = (w.window_left, w.window_right)
    out, lse = F.fwd_varlen(q, k, v, cu, w.N, w.scale, w.causal, win, sl, dropout_p,
                            dropout_seed=seed)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd_varlen(do, q, k, v, lse, D, cu, w.N, w.scale, w.causal, win, sl,
                              dropout_p, w.deterministic, dropout_seed=seed)
    torch.cuda.synchronize()
    assert F.device_status() == 0
    return (q, k, v, do), (out, lse, D, dq, dk, dv)


def compare(w, ins, outs, keep=None, keep_scale=1.0):
    q, k, v, do = (f64(t) for t in ins)
    out, lse, D, dq, dk, dv = outs
    cu = w.cu_seqlens()
    slopes = w.alibi_slopes()
    kw = dict(causal=w.causal, window_left=w.window_left, window_right=w.window_right,
              alibi_slopes=None if slopes is None else slopes.numpy(), keep=keep,
              keep_scale=keep_scale)
    o_ref, l_ref = op.packed_forward(q, k, v, cu, w.softmax_scale, **kw)
    rdq, rdk, rdv, rD = op.packed_backward(q, k, v, do, cu, w.softmax_scale, **kw)
    o_max = None
    if keep is not None and w.dtype == torch.bfloat16:
        o_max = max(1e-2, keep_scale * float(np.abs(v).max()) / 256.0)
    for b, (s, e) in enumerate(op.spans(cu)):
        if e == s:
            continue
        for h in range(w.H):
            tag = f"{w.name} seq={b} [{s},{e}) h={h}"
            check_fwd(f64(out[s:e, h]), f64(lse[h, s:e]), o_ref[s:e, h], l_ref[h, s:e],
                      w.dtype, tag, o_max=o_max)
            fl_q, fl_k = d_rounding_bounds(q[s:e, h], k[s:e, h], do[s:e, h], o_ref[s:e, h],
                                           w.softmax_scale, w.causal, w.window_left,
                                           w.window_right,
                                           None if slopes is None else float(slopes[h]))
            check_grad(f64(dq[s:e, h]), rdq[s:e, h], w.dtype, tag + " dq", floor=fl_q)
            check_grad(f64(dk[s:e, h]), rdk[s:e, h], w.dtype, tag + " dk", floor=fl_k)
            check_grad(f64(dv[s:e, h]), rdv[s:e, h], w.dtype, tag + " dv")
    # D of the GPU's own O matches the definition on the GPU's O
    ref_D = np.einsum("thd,thd->ht", f64(out), do)
    assert np.allclose(f64(D), ref_D, rtol=1e-4, atol=1e-3)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_packed_parity(w):
    ins, outs = run(w)
    compare(w, ins, outs)


@pytest.mark.parametrize("p", [0.1, 0.5])
@pytest.mark.parametrize("w", [CASES[1], CASES[2], CASES[6], CASES[7], CASES[10]],
                         ids=lambda w: w.name)
def test_packed_dropout_parity(w, p):
    seed = 4321 + w.seed
    ins, outs = run(w, p, seed)

    def keep(b, h, n):
        return philox.keep_mask(b, h, np.arange(n), n, p, seed)

    compare(w, ins, outs, keep=keep, keep_scale=philox.keep_scale(p))


@pytest.mark.parametrize("det", [False, True])
def test_packed_equals_padded_calls_bitwise(det):
    """Sequence b of a packed call equals a padded call of that sequence
    alone: the forward bit for bit (same blocks, same order), dK and dV bit for
    bit, and the deterministic dQ up to the order of its fp32 sums (the padded
    causal call adds them in its in-kernel order, the packed one in its
    second pass)."""
    w = W.packed("vs-padded", (300, 129, 0, 513, 1), H=2, d=128, causal=True, seed=83,
                 deterministic=det)
    (q, k, v, do), (out, lse, D, dq, dk, dv) = run(w, 0.25, 99)
    for b, (s, e) in enumerate(op.spans(w.cu_seqlens())):
        if e == s:
            continue
        one = [t[s:e].unsqueeze(0).contiguous() for t in (q, k, v, do)]
        # the dropout counter's batch field is the sequence index: emulate a
        # padded call at batch index b by placing the sequence at index b
        pad = [torch.zeros((b + 1,) + t.shape[1:], dtype=t.dtype, device=t.device)
               for t in one]
        for p_, t in zip(pad, one):
            p_[b] = t[0]
        o1, l1 = F.fwd(pad[0], pad[1], pad[2], causal=True, dropout_p=0.25, dropout_seed=99)
        assert torch.equal(o1[b], out[s:e]), f"seq {b}: O differs"
        assert torch.equal(l1[b], lse[:, s:e]), f"seq {b}: LSE differs"
        D1 = F.bwd_preprocess(o1, pad[3])
        g1 = F.bwd(pad[3], pad[0], pad[1], pad[2], l1, D1, causal=True, dropout_p=0.25,
                   deterministic=det, dropout_seed=99)
        torch.cuda.synchronize()
        assert torch.equal(g1[1][b], dk[s:e]) and torch.equal(g1[2][b], dv[s:e])
        if det:
            assert_same_sum_any_order(dq[s:e], g1[0][b], f"seq {b} dq")


def test_packed_mix_sampled_sequences():
    """The benchmark's length mix (32768 tokens, H=16, d=128): the shortest
    and the longest sequence on two heads, forward and backward."""
    w = W.packed_mix()
    ins, outs = run(w)
    q, k, v, do = ins
    out, lse, D, dq, dk, dv = outs
    cu = w.cu_seqlens()
    spans = op.spans(cu)
    picks = {int(np.argmin(w.lengths)), int(np.argmax(w.lengths))}
    for b in picks:
        s, e = spans[b]
        for h in (0, w.H - 1):
            sub = W.packed("one", (e - s,), H=1, d=w.d)
            sl = slice(s, e)
            args = [f64(t[sl, h:h + 1]) for t in (q, k, v)]
            o_ref, l_ref = op.packed_forward(*args, sub.cu_seqlens(), w.softmax_scale)
            check_fwd(f64(out[sl, h]), f64(lse[h, sl]), o_ref[:, 0], l_ref[0], w.dtype,
                      f"mix seq {b} h={h}")
            g = op.packed_backward(*args, f64(do[sl, h:h + 1]), sub.cu_seqlens(),
                                   w.softmax_scale)
            for got, ref, name in ((dq, g[0], "dq"), (dk, g[1], "dk"), (dv, g[2], "dv")):
                check_grad(f64(got[sl, h]), ref[:, 0], w.dtype, f"mix seq {b} h={h} {name}")


def test_autograd_packed():
    w = W.packed("ag", (200, 57), H=2, d=128, causal=True, seed=84)
    q, k, v, do = W.make_inputs(w, "cuda")
    cu = w.cu_seqlens("cuda")
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
    out = F.flash_attention_v2_varlen(qg, kg, vg, cu, w.N, causal=True)
    out.backward(do)
    o_ref, lse_ref = F.fwd_varlen(q, k, v, cu, w.N, causal=True)
    assert torch.equal(out.detach(), o_ref)
    assert torch.isfinite(qg.grad).all() and torch.isfinite(kg.grad).all()


def test_empty_batch_is_a_no_op():
    q = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    out, lse = F.fwd_varlen(q, q, q, cu, 16)
    assert out.shape == (0, 2, 128) and lse.shape == (2, 0)


def test_length_above_max_seqlen_is_reported():
    """A sequence longer than max_seqlen: every access stays inside the
    tensors (the kernels clamp the length) and the call is flagged."""
    w = W.packed("bad", (300, 200), H=1, d=128, seed=85)
    q, k, v, _ = W.make_inputs(w, "cuda")
    cu = w.cu_seqlens("cuda")
    F.fwd_varlen(q, k, v, cu, 256)   # the first sequence has 300 rows
    torch.cuda.synchronize()
    assert F.device_status() == F.STATUS_BAD_SEQLENS
    assert F.device_status() == 0    # cleared by the read
