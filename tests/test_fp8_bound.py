"""The e4m3 forward's error bound (tests/helpers.fp8_o_bound) checked on the
CPU against a model of the kernel's rounding.

The model follows the kernel's arithmetic where it rounds:
- blocks of 128 keys in order;
- a running max that moves only when a block's max exceeds it by more than
  8 (base 2);
- P = 2^(x - m) kept in full precision for the row sum, and rounded to e4m3
  (round to nearest even) for the PV product;
- O divided by l once at the end, then rounded to bf16.

Everything else runs in float64.  The bound must hold for every element. It
must also not be loose: over the cases, the worst element uses more than
half of it.  A bound that drops the e4m3 rounding term fails.
"""

import numpy as np
import pytest
import torch

from exact_attention_147_b200 import workloads as W
from oracle import attention as oa
from tests.helpers import fp8_o_bound

LOG2E = 1.0 / np.log(2.0)


def _e4m3(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32).to(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32).to(
        torch.bfloat16).to(torch.float64).numpy()


def model_forward(q, k, v, scale, causal=False, wl=-1, wr=-1, slope=None, block=128, tau=8.0):
    n = q.shape[0]
    x = oa.head_scores(q, k, np.arange(n), scale, causal, wl, wr, slope) * LOG2E
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    o = np.zeros((n, v.shape[1]))
    for j0 in range(0, k.shape[0], block):
        xb = x[:, j0:j0 + block]
        mx = xb.max(axis=1)
        grow = mx > m + tau
        with np.errstate(invalid="ignore"):  # -inf - -inf in rows that saw no key yet
            alpha = np.where(grow, np.exp2(np.where(np.isfinite(m), m - mx, -np.inf)), 1.0)
        m = np.where(grow, mx, m)
        m_use = np.where(np.isfinite(m), m, 0.0)
        p = np.exp2(xb - m_use[:, None])
        l = l * alpha + p.sum(axis=1)
        o = o * alpha[:, None] + _e4m3(p) @ v[j0:j0 + block]
    out = np.where(l[:, None] > 0, o / np.where(l > 0, l, 1.0)[:, None], 0.0)
    return _bf16(out)


CASES = [
    W.Workload("n300", B=1, N=300, H=1, d=128, seed=211),
    W.Workload("n513-causal", B=1, N=513, H=1, d=128, causal=True, seed=212),
    W.Workload("window", B=1, N=700, H=1, d=128, causal=True, window_left=130, window_right=0,
               seed=215),
    W.Workload("alibi", B=1, N=520, H=1, d=128, causal=True, alibi=True, seed=217),
    W.Workload("big-logits", B=1, N=640, H=1, d=128, q_std=3.0, k_std=3.0, seed=218),
    W.Workload("small-v", B=1, N=384, H=1, d=128, v_std=0.01, seed=219, scale=0.05),
]


def _case(w):
    q8, k8, v8, (qd, kd, vd) = W.make_fp8_inputs(w)
    q, k, v = (t[0, :, 0].to(torch.float64).numpy() * s for t, s in ((q8, qd), (k8, kd), (v8, vd)))
    slopes = w.alibi_slopes()
    slope = None if slopes is None else float(slopes[0])
    args = (w.softmax_scale, w.causal, w.window_left, w.window_right, slope)
    o_ref, _ = oa.head_forward(q, k, v, *args)
    return q, k, v, args, o_ref


def _worst_ratio(w):
    q, k, v, args, o_ref = _case(w)
    err = np.abs(model_forward(q, k, v, *args) - o_ref)
    return float((err / fp8_o_bound(q, k, v, *args)).max())


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_bound_covers_the_rounding_model(w):
    assert _worst_ratio(w) <= 1.0


def test_bound_is_not_loose():
    # the worst element over the cases uses more than half of its bound
    assert max(_worst_ratio(w) for w in CASES) > 0.5


def test_bound_without_the_e4m3_term_is_exceeded():
    q, k, v, args, o_ref = _case(CASES[0])
    err = np.abs(model_forward(q, k, v, *args) - o_ref)
    o = np.abs(o_ref)
    assert (err > 2.0 ** -8 * o + 1e-6 * np.abs(v).max()).any()
