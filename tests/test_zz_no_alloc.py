"""fa2_bwd_noalloc: the backward pass for callers that cannot allocate.

Callers such as a framework that owns all device memory through its own
pool, or a plugin interface that supplies no workspace, cannot call
cudaMalloc when they run the backward pass.  fa2_bwd_noalloc takes its fp32
dQ accumulator from a fixed array inside the library instead.  These tests
call it through the C ABI and compare it with fa2_bwd, which uses a
caller-provided workspace.  (This file is collected last on purpose.)
"""

import ctypes

import pytest
import torch

from exact_attention_147_b200 import build as fa2_build
from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W
from tests.helpers import check_grad, f64


def _lib():
    fa2_build.build()
    return F.load_library()


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _lib()
    P = ctypes.c_void_p(0x100000)
    s = F.Strides(2048 * 16 * 128, 16 * 128, 128)
    # B*H*N*d = 8*16*2048*128 floats, far above the fixed scratch
    st = lib.fa2_bwd_noalloc(P, P, P, P, P, P, ctypes.c_void_p(0x200000),
                             ctypes.c_void_p(0x300000), ctypes.c_void_p(0x400000),
                             8, 2048, 16, 128, s, s, s, s, s, s, s, 0.0, 0, -1, -1, None, 0.0,
                             None)
    assert st == F.FA2_ERR_SCRATCH_LIMIT
    assert "scratch" in F.strerror(st)


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_on_two_calls():
    lib = _lib()
    w = W.Workload("noalloc", B=2, N=300, H=4, d=128, causal=True, seed=41)
    assert w.B * w.H * w.N * w.d <= F.NOALLOC_MAX_DQ_FLOATS
    q, k, v, do = W.make_inputs(w, "cuda")
    out, lse = F.fwd(q, k, v, causal=True)
    D = F.bwd_preprocess(out, do)
    rdq, rdk, rdv = F.bwd(do, q, k, v, lse, D, causal=True, deterministic=False)
    torch.cuda.synchronize()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st_ = F._strides
    for call in range(2):   # the second call must not see the first one's sums
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        status = lib.fa2_bwd_noalloc(
            F._ptr(q), F._ptr(k), F._ptr(v), F._ptr(do), F._ptr(lse), F._ptr(D), F._ptr(dq),
            F._ptr(dk), F._ptr(dv), w.B, w.N, w.H, w.d, st_(q), st_(k), st_(v), st_(do),
            st_(dq), st_(dk), st_(dv), 0.0, 1, -1, -1, None, 0.0, stream)
        assert status == F.FA2_OK, F.strerror(status)
        torch.cuda.synchronize()
        assert F.device_status() == 0
        for got, ref, name in ((dq, rdq, "dq"), (dk, rdk, "dk"), (dv, rdv, "dv")):
            check_grad(f64(got), f64(ref), w.dtype, f"noalloc call {call} {name}")
