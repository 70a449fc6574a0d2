"""FP8 (e4m3) forward: libfa2 against the fp64 oracle on the dequantised
inputs.

The oracle computes exact attention of q_descale * q8, k_descale * k8,
v_descale * v8.  The kernel's only approximation is P rounded to e4m3
before the PV product (plus bf16 rounding of O); the bound of that error is
derived per element in tests/helpers.fp8_o_bound and checked element by
element, with LSE (computed from the exact fp32 scores) at 1e-3.
"""

import numpy as np
import pytest
import torch

from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W
from oracle import attention as oa
from tests.helpers import f64, fp8_o_bound

pytestmark = pytest.mark.gpu


def run_and_check(w, heads=None):
    q8, k8, v8, (qd, kd, vd) = W.make_fp8_inputs(w, "cuda")
    slopes = w.alibi_slopes()
    sl = None if slopes is None else slopes.cuda()
    out, lse = F.fwd_fp8(q8, k8, v8, qd, kd, vd, w.scale, w.causal,
                         (w.window_left, w.window_right), sl)
    torch.cuda.synchronize()
    assert F.device_status() == 0
    assert out.dtype == torch.bfloat16
    pairs = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    worst = 0.0
    for b, h in pairs:
        q = f64(q8[b, :, h]) * qd
        k = f64(k8[b, :, h]) * kd
        v = f64(v8[b, :, h]) * vd
        slope = None if slopes is None else float(slopes[h])
        o_ref, l_ref = oa.head_forward(q, k, v, w.softmax_scale, w.causal, w.window_left,
                                       w.window_right, slope)
        bound = fp8_o_bound(q, k, v, w.softmax_scale, w.causal, w.window_left, w.window_right,
                            slope)
        got = f64(out[b, :, h])
        err = np.abs(got - o_ref)
        tag = f"{w.name} ({b},{h})"
        assert np.isfinite(got).all(), tag
        over = err > bound
        assert not over.any(), (f"{tag}: O err {err[over].max():.3e} over the e4m3 bound at "
                                f"{np.argwhere(over)[0]}")
        assert np.abs(f64(lse[b, h]) - l_ref).max() <= 1e-3, tag + " LSE"
        worst = max(worst, float((err / np.maximum(bound, 1e-30)).max()))
    return worst


CASES = [
    W.Workload("fp8-n300", B=2, N=300, H=2, d=128, seed=111),
    W.Workload("fp8-n513-causal", B=1, N=513, H=2, d=128, causal=True, seed=112),
    W.Workload("fp8-n1", B=1, N=1, H=2, d=128, seed=113),
    W.Workload("fp8-n129", B=2, N=129, H=1, d=128, causal=True, seed=114),
    W.Workload("fp8-window", B=1, N=700, H=2, d=128, causal=True, window_left=130,
               window_right=0, seed=115),
    W.Workload("fp8-window-both", B=1, N=600, H=2, d=128, window_left=5, window_right=7, seed=116),
    W.Workload("fp8-alibi", B=1, N=520, H=4, d=128, causal=True, alibi=True, seed=117),
    W.Workload("fp8-big-logits", B=1, N=640, H=2, d=128, q_std=3.0, k_std=3.0, seed=118),
    W.Workload("fp8-small-v", B=1, N=384, H=2, d=128, v_std=0.01, seed=119, scale=0.05),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fp8_parity(w):
    run_and_check(w)


def test_fp8_bench_workload_sampled_heads():
    for causal in (False, True):
        run_and_check(W.mid(causal).replace(name="fp8-mid"), heads=[(0, 0), (3, 7), (7, 15)])


def test_fp8_is_deterministic():
    w = W.Workload("fp8-det", B=2, N=700, H=2, d=128, causal=True, seed=120)
    q8, k8, v8, (qd, kd, vd) = W.make_fp8_inputs(w, "cuda")
    o1, l1 = F.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=True)
    o2, l2 = F.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fp8_rejects_other_head_dims():
    w = W.Workload("fp8-d64", B=1, N=128, H=1, d=64, seed=121)
    q8, k8, v8, (qd, kd, vd) = W.make_fp8_inputs(w, "cuda")
    with pytest.raises(F.Fa2Error) as e:
        F.fwd_fp8(q8, k8, v8, qd, kd, vd)
    assert e.value.status == F.FA2_ERR_UNSUPPORTED
