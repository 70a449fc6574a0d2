"""The bounded-wait path on the GPU: a wait that runs out must end the
kernel with an error status, not a hang, and leave the library usable.

fa2_test_skip_arrive (a test switch, off by default) makes the first CTA of
a launch withhold one mbarrier arrive, so the MMA warp's wait for it runs
out after the limit set by fa2_set_wait_limit_ms.  The call must then report
FA2_ERR_DEVICE_TIMEOUT with a site code of the kernel that gave up, every
other role of that CTA must wind down through its abort flag (the test would
time out otherwise), and the next normal call -- on the same stream, so on
the same work-counter pair for the counter-scheduled (packed) calls -- must
match the fp64 oracle.
"""

import numpy as np
import pytest
import torch

from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W
from oracle import attention as oa
from tests.helpers import check_fwd, check_grad, f64, oracle_head_bwd, oracle_head_fwd

pytestmark = pytest.mark.gpu

# site codes: forward 0x1xx-0x4xx (producer, MMA, softmax/epilogue, drain),
# dK/dV kernel 0x5xx-0x8xx (producer, MMA, compute, dQ drain)
FWD_SITES = range(0x100, 0x500)
BWD_SITES = range(0x500, 0x900)


@pytest.fixture
def short_waits():
    F.device_status(clear=True)
    F.set_wait_limit_ms(20)
    yield
    F.test_skip_arrive(0)
    F.set_wait_limit_ms(1000)
    F.device_status(clear=True)


def _padded_ref(w, q, k, v, do, b, h):
    return oracle_head_fwd(w, q, k, v, b, h), oracle_head_bwd(w, q, k, v, do, b, h)


@pytest.mark.parametrize("d", [128, 64])
def test_forward_wait_runs_out_then_recovers(short_waits, d):
    w = W.Workload("timeout-fwd", B=2, N=1024, H=4, d=d, causal=True, seed=131)
    q, k, v, do = W.make_inputs(w, "cuda")
    F.test_skip_arrive(1)
    F.fwd(q, k, v, causal=True)
    code = F.device_status(clear=True)
    assert code in FWD_SITES, hex(code)
    F.test_skip_arrive(0)
    out, lse = F.fwd(q, k, v, causal=True)
    assert F.device_status(clear=True) == 0
    for b, h in [(0, 0), (1, 3)]:
        (o_ref, l_ref), _ = _padded_ref(w, q, k, v, do, b, h)
        check_fwd(f64(out[b, :, h]), f64(lse[b, h]), o_ref, l_ref, w.dtype, f"({b},{h})")


def test_backward_wait_runs_out_then_recovers(short_waits):
    w = W.Workload("timeout-bwd", B=1, N=768, H=4, d=128, seed=132)
    q, k, v, do = W.make_inputs(w, "cuda")
    out, lse = F.fwd(q, k, v)
    D = F.bwd_preprocess(out, do)
    F.test_skip_arrive(2)
    F.bwd(do, q, k, v, lse, D)
    code = F.device_status(clear=True)
    assert code in BWD_SITES, hex(code)
    F.test_skip_arrive(0)
    dq, dk, dv = F.bwd(do, q, k, v, lse, D)
    assert F.device_status(clear=True) == 0
    for b, h in [(0, 0), (0, 3)]:
        _, (rdq, rdk, rdv, _) = _padded_ref(w, q, k, v, do, b, h)
        check_grad(f64(dq[b, :, h]), rdq, w.dtype, "dq")
        check_grad(f64(dk[b, :, h]), rdk, w.dtype, "dk")
        check_grad(f64(dv[b, :, h]), rdv, w.dtype, "dv")


def test_packed_abort_leaves_the_counter_pair_usable(short_waits):
    # The aborted CTA stops taking units; the pair it shares with the rest of
    # the call must still be back at zero (and is cleared before every launch
    # anyway) so the next packed calls on this stream do all their work.
    w = W.packed("timeout-packed", (700, 129, 1, 300, 513), H=2, d=128, causal=True, seed=133)
    q, k, v, do = W.make_inputs(w, "cuda")
    cu = w.cu_seqlens("cuda")
    for which in (1, 2):
        F.test_skip_arrive(which)
        o, l = F.fwd_varlen(q, k, v, cu, w.N, causal=True)
        D = F.bwd_preprocess(o, do)
        F.bwd_varlen(do, q, k, v, l, D, cu, w.N, causal=True)
        code = F.device_status(clear=True)
        assert code in (FWD_SITES if which == 1 else BWD_SITES), hex(code)
    F.test_skip_arrive(0)
    out, lse = F.fwd_varlen(q, k, v, cu, w.N, causal=True)
    D = F.bwd_preprocess(out, do)
    dq, dk, dv = F.bwd_varlen(do, q, k, v, lse, D, cu, w.N, causal=True)
    assert F.device_status(clear=True) == 0
    starts = np.concatenate([[0], np.cumsum(w.lengths)])
    for si, n in enumerate(w.lengths):
        if n == 0:
            continue
        r = slice(int(starts[si]), int(starts[si]) + n)
        for h in range(w.H):
            args = (f64(q[r, h]), f64(k[r, h]), f64(v[r, h]))
            o_ref, l_ref = oa.head_forward(*args, w.softmax_scale, True)
            check_fwd(f64(out[r, h]), f64(lse[h, r]), o_ref, l_ref, w.dtype, f"seq {si} h {h}")
            rdq, rdk, rdv, _ = oa.head_backward(*args, f64(do[r, h]), w.softmax_scale, True)
            check_grad(f64(dk[r, h]), rdk, w.dtype, "dk")
            check_grad(f64(dv[r, h]), rdv, w.dtype, "dv")
