"""Backward parity: D, dQ, dK, dV from libfa2 against the fp64 oracle.

The GPU runs its own forward (for LSE and O), bwd_preprocess and bwd; the
oracle recomputes every gradient from the same inputs.
"""

import dataclasses

import numpy as np
import pytest
import torch

from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W
from oracle import attention as oa
from tests.helpers import check_grad, f64, oracle_head_bwd

pytestmark = pytest.mark.gpu


def run_fwd_bwd(w, q, k, v, do, deterministic=None):
    det = w.deterministic if deterministic is None else deterministic
    slopes = w.alibi_slopes()
    slopes = None if slopes is None else slopes.cuda()
    win = (w.window_left, w.window_right)
    out, lse = F.fwd(q, k, v, w.scale, w.causal, win, slopes)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd(do, q, k, v, lse, D, w.scale, w.causal, win, slopes, 0.0, det)
    torch.cuda.synchronize()
    assert F.device_status() == 0
    return out, D, dq, dk, dv


def compare_heads(w, heads, det=None):
    q, k, v, do = W.make_inputs(w, "cuda")
    out, D, dq, dk, dv = run_fwd_bwd(w, q, k, v, do, det)
    for b, h in heads:
        # D against the oracle's definition applied to the GPU's own O
        d_ref = oa.bwd_preprocess(f64(out[b:b + 1, :, h:h + 1]), f64(do[b:b + 1, :, h:h + 1]))
        assert np.abs(f64(D[b, h]) - d_ref[0, 0]).max() <= 1e-4 * max(1.0, np.abs(d_ref).max())
        rdq, rdk, rdv, _ = oracle_head_bwd(w, q, k, v, do, b, h)
        tag = f"{w.name} ({b},{h})"
        check_grad(f64(dq[b, :, h]), rdq, w.dtype, tag + " dq")
        check_grad(f64(dk[b, :, h]), rdk, w.dtype, tag + " dk")
        check_grad(f64(dv[b, :, h]), rdv, w.dtype, tag + " dv")
    return dq, dk, dv


SMALL = []
for n in (1, 127, 129, 300, 513):
    for d in (64, 128):
        SMALL.append(W.Workload(f"small-n{n}-d{d}", B=2, N=n, H=2, d=d, seed=n + d))
        SMALL.append(W.Workload(f"small-n{n}-d{d}-causal", B=2, N=n, H=2, d=d, causal=True,
                                seed=n + d + 1))
SMALL += [
    W.Workload("win-130-0", B=1, N=700, H=2, d=128, causal=True, window_left=130,
               window_right=0, seed=11),
    W.Workload("win-5-7", B=1, N=600, H=2, d=64, window_left=5, window_right=7, seed=12),
    W.Workload("win-0-0", B=1, N=300, H=1, d=128, window_left=0, window_right=0, seed=13),
    W.Workload("alibi-causal", B=2, N=520, H=4, d=128, causal=True, alibi=True, seed=16),
    W.Workload("alibi-noncausal", B=1, N=390, H=3, d=64, alibi=True, seed=17),
    W.Workload("alibi-window", B=1, N=700, H=2, d=128, causal=True, alibi=True,
               window_left=200, window_right=0, seed=18),
    W.Workload("big-logits-causal", B=1, N=640, H=2, d=64, causal=True, q_std=4.0, k_std=4.0,
               seed=20),
    W.Workload("det-small", B=2, N=400, H=2, d=128, causal=True, deterministic=True, seed=24),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_full(w):
    compare_heads(w, [(b, h) for b in range(w.B) for h in range(w.H)])


@pytest.mark.parametrize("w", [W.tiny(False), W.tiny(True), W.tiny(False, True),
                               W.tiny(True, True)], ids=lambda w: w.name)
def test_tiny_fp32(w):
    compare_heads(w, [(0, 0), (0, 1)])


@pytest.mark.parametrize("causal", [False, True])
def test_mid_sampled(causal):
    w = W.mid(causal)
    compare_heads(w, [(0, 0), (w.B - 1, w.H - 1)])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", W.SWEEP_N)
@pytest.mark.parametrize("d", [128, 64])
def test_sweep_sampled(n, d, causal):
    # every point of the sequence-length sweep (hidden 2048 as H=16 x d=128
    # and as H=32 x d=64), one whole head each
    w = W.sweep(n, d, causal)
    compare_heads(w, [(w.B - 1, w.H - 1)])


@pytest.mark.parametrize("d", [128, 64])
def test_causal_long_sampled(d):
    # 128 key blocks under a causal mask: the dK/dV kernel takes its items
    # from the shared counter (both head dims), first and last heads
    w = W.sweep(16384, d, causal=True)
    compare_heads(w, [(0, 0), (0, w.H - 1)])


@pytest.mark.parametrize("n,causal", [(1024, False), (4096, True), (16384, True)])
def test_deterministic_d64(n, causal):
    # the padded-layout ordered dQ pass at d = 64: parity on a sampled head
    # and bitwise-identical dq, dk, dv across two runs
    w = dataclasses.replace(W.sweep(n, 64, causal), deterministic=True)
    dq1, dk1, dv1 = compare_heads(w, [(w.B - 1, w.H - 1)])
    q, k, v, do = W.make_inputs(w, "cuda")
    _, _, dq2, dk2, dv2 = run_fwd_bwd(w, q, k, v, do)
    assert torch.equal(dq1, dq2) and torch.equal(dk1, dk2) and torch.equal(dv1, dv2)


def test_long_local_sampled():
    w = W.long_local()
    compare_heads(w, [(0, 31)])


def test_alibi_deterministic():
    """Config with ALiBi + deterministic backward: parity on sampled heads and
    bitwise-identical dq, dk, dv across two runs."""
    w = W.alibi_det()
    dq1, dk1, dv1 = compare_heads(w, [(0, 0), (3, 15)])
    q, k, v, do = W.make_inputs(w, "cuda")
    _, _, dq2, dk2, dv2 = run_fwd_bwd(w, q, k, v, do)
    assert torch.equal(dq1, dq2) and torch.equal(dk1, dk2) and torch.equal(dv1, dv2)


def test_autograd_function():
    w = W.Workload("autograd", B=1, N=300, H=2, d=128, causal=True, seed=31)
    q, k, v, do = W.make_inputs(w, "cuda")
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
    out = F.flash_attention_v2(qg, kg, vg, causal=True)
    out.backward(do)
    for b in range(w.B):
        for h in range(w.H):
            rdq, rdk, rdv, _ = oracle_head_bwd(w, q, k, v, do, b, h)
            check_grad(f64(qg.grad[b, :, h]), rdq, w.dtype, "autograd dq")
            check_grad(f64(kg.grad[b, :, h]), rdk, w.dtype, "autograd dk")
            check_grad(f64(vg.grad[b, :, h]), rdv, w.dtype, "autograd dv")
