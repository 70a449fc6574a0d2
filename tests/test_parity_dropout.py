"""Dropout parity: libfa2's dropout mask and gradients against the oracle.

The mask itself is compared bit for bit: with q = 0 every visible key gets
the same probability 1/N, so when value row j is the unit vector e_(j mod d)
for the keys of one half of the sequence and zero for the other half, output
element (i, c) is keep(i, j) / N times the keep scale for the single key j
of that half with j mod d = c (forward); one-hot dO rows over one half of
the queries do the same for dV (backward key-row kernel).  Each half is its
own call, so every element of the mask is read on its own.  Outputs and
gradients are then compared with the fp64 oracle, which draws the same mask
with its own Philox4x32-10 (pinned to the generator's published
known-answer vectors in tests/test_oracle_dropout.py).
"""

import numpy as np
import pytest
import torch

from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W
from oracle import attention as oa
from oracle import philox
from tests.helpers import assert_same_sum_any_order, check_fwd, check_grad, d_rounding_bounds, f64

pytestmark = pytest.mark.gpu


def onehot_half(n, d, half, dtype):
    """[n, d]: row j is e_(j mod d) for the rows of half `half` (d rows each),
    zero elsewhere."""
    v = torch.zeros(n, d)
    rows = torch.arange(half * d, (half + 1) * d)
    v[rows, rows % d] = 1.0
    return v.to(dtype)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("p,seed", [(0.5, 11), (0.1, 2**40 + 7), (0.99, 5)])
def test_mask_bits_forward_and_backward(dtype, p, seed, d):
    B, N, H = 2, 256, 3
    q = torch.zeros(B, N, H, d, dtype=dtype, device="cuda")
    g = torch.Generator().manual_seed(3)
    k = torch.randn(B, N, H, d, generator=g).to(dtype).cuda()
    ks = philox.keep_scale(p)
    keep = {(b, h): philox.keep_mask(b, h, np.arange(N), N, p, seed).astype(np.float64)
            for b in range(B) for h in range(H)}
    for half in range(N // d):
        base = onehot_half(N, d, half, dtype)
        sl = slice(half * d, (half + 1) * d)
        # value rows of keys in this half only: O[i, c] = ks / N * keep[i, half*d + c]
        v = base[None, :, None, :].expand(B, N, H, d).contiguous().cuda()
        out, lse = F.fwd(q, k, v, dropout_p=p, dropout_seed=seed)
        # dO rows of queries in this half only: dV[j, c] = ks / N * keep[half*d + c, j]
        do = base[None, :, None, :].expand(B, N, H, d).contiguous().cuda()
        D = F.bwd_preprocess(out, do)
        dq, dk, dv = F.bwd(do, q, k, v, lse, D, dropout_p=p, dropout_seed=seed)
        torch.cuda.synchronize()
        assert F.device_status() == 0
        for b in range(B):
            for h in range(H):
                m = keep[(b, h)]
                got_f = np.rint(f64(out[b, :, h]) * N / ks)
                assert np.array_equal(got_f, m[:, sl]), f"forward mask b={b} h={h} half={half}"
                got_b = np.rint(f64(dv[b, :, h]) * N / ks)
                assert np.array_equal(got_b, m[sl, :].T), f"backward mask b={b} h={h} half={half}"


CASES = [
    W.Workload("drop-n300-d128", B=2, N=300, H=2, d=128, seed=51),
    W.Workload("drop-n300-d128-causal", B=1, N=300, H=2, d=128, causal=True, seed=52),
    W.Workload("drop-n513-d64", B=1, N=513, H=2, d=64, seed=53),
    W.Workload("drop-alibi-window", B=1, N=400, H=2, d=128, causal=True, alibi=True,
               window_left=150, window_right=0, seed=54),
    W.Workload("drop-det", B=1, N=384, H=2, d=128, causal=True, deterministic=True, seed=55),
    W.Workload("drop-fp32", B=1, N=256, H=2, d=64, dtype=torch.float32, causal=True, seed=56,
               scale=1.0 / 8.0),
    # units of a single key block (the mask ring's first entry is its only one)
    W.Workload("drop-n1-d128", B=2, N=1, H=2, d=128, seed=58),
    W.Workload("drop-n128-d64-causal", B=1, N=128, H=2, d=64, causal=True, seed=59),
]


@pytest.mark.parametrize("p", [0.1, 0.5])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_dropout_parity(w, p):
    seed = 1234 + w.seed
    q, k, v, do = W.make_inputs(w, "cuda")
    slopes = w.alibi_slopes()
    sl = None if slopes is None else slopes.cuda()
    win = (w.window_left, w.window_right)
    out, lse = F.fwd(q, k, v, w.scale, w.causal, win, sl, p, dropout_seed=seed)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd(do, q, k, v, lse, D, w.scale, w.causal, win, sl, p, w.deterministic,
                       dropout_seed=seed)
    torch.cuda.synchronize()
    assert F.device_status() == 0
    ks = philox.keep_scale(p)
    for b in range(w.B):
        for h in range(w.H):
            keep = philox.keep_mask(b, h, np.arange(w.N), w.N, p, seed)
            slope = None if slopes is None else float(slopes[h])
            args = (f64(q[b, :, h]), f64(k[b, :, h]), f64(v[b, :, h]))
            o_ref, l_ref = oa.head_forward(*args, w.softmax_scale, w.causal, w.window_left,
                                           w.window_right, slope, keep=keep, keep_scale=ks)
            # the dropped output has a larger range; bf16 rounding scales with it
            o_max = None
            if w.dtype == torch.bfloat16:
                o_max = max(1e-2, ks * float(v[b, :, h].abs().max()) / 256.0)
            check_fwd(f64(out[b, :, h]), f64(lse[b, h]), o_ref, l_ref, w.dtype,
                      f"{w.name} p={p} ({b},{h})", o_max=o_max)
            rdq, rdk, rdv, _ = oa.head_backward(*args, f64(do[b, :, h]), w.softmax_scale,
                                                w.causal, w.window_left, w.window_right, slope,
                                                keep=keep, keep_scale=ks)
            tag = f"{w.name} p={p} ({b},{h})"
            # D comes from the bf16 output: where the exact dQ / dK cancel (a
            # query that sees one key, N=1), what remains is that rounding
            fq = fk = 0.0
            if w.dtype == torch.bfloat16:
                fq, fk = d_rounding_bounds(args[0], args[1], f64(do[b, :, h]), o_ref,
                                           w.softmax_scale, w.causal, w.window_left,
                                           w.window_right, slope)
            check_grad(f64(dq[b, :, h]), rdq, w.dtype, tag + " dq", floor=fq)
            check_grad(f64(dk[b, :, h]), rdk, w.dtype, tag + " dk", floor=fk)
            check_grad(f64(dv[b, :, h]), rdv, w.dtype, tag + " dv")


def test_dropout_mid_sampled_heads():
    w = W.mid(False)
    p, seed = 0.1, 99
    q, k, v, do = W.make_inputs(w, "cuda")
    out, lse = F.fwd(q, k, v, dropout_p=p, dropout_seed=seed)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd(do, q, k, v, lse, D, dropout_p=p, dropout_seed=seed)
    torch.cuda.synchronize()
    ks = philox.keep_scale(p)
    for b, h in [(0, 0), (7, 15)]:
        keep = philox.keep_mask(b, h, np.arange(w.N), w.N, p, seed)
        args = (f64(q[b, :, h]), f64(k[b, :, h]), f64(v[b, :, h]))
        o_ref, l_ref = oa.head_forward(*args, w.softmax_scale, keep=keep, keep_scale=ks)
        check_fwd(f64(out[b, :, h]), f64(lse[b, h]), o_ref, l_ref, w.dtype, f"mid ({b},{h})")
        rdq, rdk, rdv, _ = oa.head_backward(*args, f64(do[b, :, h]), w.softmax_scale,
                                            keep=keep, keep_scale=ks)
        check_grad(f64(dq[b, :, h]), rdq, w.dtype, "mid dq")
        check_grad(f64(dk[b, :, h]), rdk, w.dtype, "mid dk")
        check_grad(f64(dv[b, :, h]), rdv, w.dtype, "mid dv")


def test_autograd_draws_fresh_masks():
    w = W.Workload("ag-drop", B=1, N=256, H=2, d=128, seed=61)
    q, k, v, do = W.make_inputs(w, "cuda")
    o1 = F.flash_attention_v2(q, k, v, dropout_p=0.3)
    o2 = F.flash_attention_v2(q, k, v, dropout_p=0.3)
    assert not torch.equal(o1, o2)
    qg = q.clone().requires_grad_(True)
    F.flash_attention_v2(qg, k, v, dropout_p=0.3).backward(do)
    assert torch.isfinite(qg.grad).all()


@pytest.mark.parametrize("d", [128, 64])
def test_threshold_zero_keeps_everything(d):
    # p < 0.5/256 rounds the byte threshold to 0: every byte passes and the
    # keep scale is 256/256, so the dropout kernels must give exactly what
    # the kernels without dropout give.
    w = W.Workload("drop-t0", B=1, N=384, H=2, d=d, causal=True, seed=57)
    q, k, v, do = W.make_inputs(w, "cuda")
    ref = F.fwd(q, k, v, causal=True)
    got = F.fwd(q, k, v, causal=True, dropout_p=1e-3, dropout_seed=3)
    D = F.bwd_preprocess(ref[0], do)
    gref = F.bwd(do, q, k, v, ref[1], D, causal=True)
    ggot = F.bwd(do, q, k, v, ref[1], D, causal=True, dropout_p=1e-3, dropout_seed=3)
    torch.cuda.synchronize()
    assert F.device_status() == 0
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    for a, b in zip(ggot, gref):
        assert_same_sum_any_order(a, b)
