"""The C ABI without a GPU: the library loads, exports every symbol its
header declares, and rejects invalid arguments before touching CUDA."""

import ctypes
import os
import re

import pytest
import torch

from exact_attention_147_b200 import build as fa2_build
from exact_attention_147_b200 import fa2 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa2.h")


@pytest.fixture(scope="module")
def lib():
    fa2_build.build()
    return F.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa2_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(F.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n


def test_strerror(lib):
    for code in range(5):
        assert F.strerror(code).startswith("FA2_")
    assert "unknown" in F.strerror(99)


# Fake, 16-byte aligned device addresses: every call below fails its argument
# checks, so nothing dereferences them.
P = ctypes.c_void_p(0x100000)
S128 = F.Strides(8 * 2048 * 16 * 128 // 8, 16 * 128, 128)   # [B,N,H,d] dense strides


def call_fwd(lib, **kw):
    a = dict(q=P, k=P, v=P, o=ctypes.c_void_p(0x200000), lse=P, B=1, N=256, H=2, d=128,
             dtype=F.FA2_BF16, s=S128, scale=0.0, causal=0, wl=-1, wr=-1, alibi=None,
             dropout=0.0)
    a.update(kw)
    return lib.fa2_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["N"], a["H"], a["d"],
                       a["dtype"], a["s"], a["s"], a["s"], a["s"], a["scale"], a["causal"],
                       a["wl"], a["wr"], a["alibi"], a["dropout"], 0, None)


@pytest.mark.parametrize("bad", [
    dict(q=None), dict(k=None), dict(lse=None), dict(d=96), dict(d=0), dict(N=0), dict(B=0),
    dict(H=-1), dict(dtype=7), dict(q=ctypes.c_void_p(0x100008)),
    dict(s=F.Strides(8, 12, 128)), dict(s=F.Strides(0, 128, 128)), dict(scale=float("nan")),
    dict(dropout=float("nan")), dict(dropout=1.5), dict(dropout=0.999), dict(dropout=-0.1),
    dict(alibi=ctypes.c_void_p(0x100002)),
    dict(o=P),  # output aliases an input
])
def test_fwd_rejects_invalid(lib, bad):
    assert call_fwd(lib, **bad) == F.FA2_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_call_without_device_is_cuda_error(lib):
    assert call_fwd(lib) == F.FA2_ERR_CUDA
    assert call_fwd(lib, dropout=0.25) == F.FA2_ERR_CUDA   # a valid dropout probability


def test_preprocess_and_bwd_reject_invalid(lib):
    s = S128
    assert lib.fa2_bwd_preprocess(P, P, None, 1, 256, 2, 128, F.FA2_BF16, s, s, None) == \
        F.FA2_ERR_INVALID_ARG
    assert lib.fa2_bwd_preprocess(P, P, P, 1, 256, 2, 100, F.FA2_BF16, s, s, None) == \
        F.FA2_ERR_INVALID_ARG
    need = lib.fa2_bwd_workspace_size(1, 256, 2, 128, F.FA2_BF16, 0)
    # workspace too small
    st = lib.fa2_bwd(P, P, P, P, P, P, ctypes.c_void_p(0x300000), ctypes.c_void_p(0x400000),
                     ctypes.c_void_p(0x500000), ctypes.c_void_p(0x600000), need - 1,
                     1, 256, 2, 128, F.FA2_BF16, s, s, s, s, s, s, s, 0.0, 0, -1, -1, None,
                     0.0, 0, 0, None)
    assert st == F.FA2_ERR_INVALID_ARG
    # dropout probability whose byte threshold would keep nothing
    st = lib.fa2_bwd(P, P, P, P, P, P, ctypes.c_void_p(0x300000), ctypes.c_void_p(0x400000),
                     ctypes.c_void_p(0x500000), ctypes.c_void_p(0x600000), need,
                     1, 256, 2, 128, F.FA2_BF16, s, s, s, s, s, s, s, 0.0, 0, -1, -1, None,
                     0.999, 0, 0, None)
    assert st == F.FA2_ERR_INVALID_ARG


def test_workspace_size(lib):
    assert lib.fa2_bwd_workspace_size(2, 300, 3, 64, F.FA2_BF16, 0) == 2 * 300 * 3 * 64 * 4
    assert lib.fa2_bwd_workspace_size(1, 256, 2, 64, F.FA2_F32, 0) == 0
    assert lib.fa2_bwd_workspace_size(1, 256, 2, 96, F.FA2_BF16, 0) == 0


def test_wait_limit(lib):
    assert lib.fa2_set_wait_limit_ms(0) == F.FA2_ERR_INVALID_ARG
    assert lib.fa2_set_wait_limit_ms(1000) == F.FA2_OK


# ----------------------------------------------------------------- packed batches
CU = ctypes.c_void_p(0x700000)          # fake, 4-byte aligned device offsets
SP = F.Strides(0, 16 * 128, 128)        # [total, H=16, d=128] packed strides


def call_fwd_varlen(lib, **kw):
    a = dict(q=P, k=P, v=P, o=ctypes.c_void_p(0x200000), lse=P, cu=CU, B=3, max_seqlen=512,
             total=1000, H=16, d=128, dtype=F.FA2_BF16, s=SP, dropout=0.0)
    a.update(kw)
    return lib.fa2_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu"], a["B"],
                              a["max_seqlen"], a["total"], a["H"], a["d"], a["dtype"], a["s"],
                              a["s"], a["s"], a["s"], 0.0, 0, -1, -1, None, a["dropout"], 0, None)


@pytest.mark.parametrize("bad", [
    dict(cu=None), dict(cu=ctypes.c_void_p(0x700002)), dict(max_seqlen=0), dict(total=-1),
    dict(B=0), dict(d=96), dict(q=None), dict(s=F.Strides(0, 12, 128)), dict(o=P),
    dict(dropout=1.0), dict(s=F.Strides(0, 1 << 37, 128)),
])
def test_fwd_varlen_rejects_invalid(lib, bad):
    assert call_fwd_varlen(lib, **bad) == F.FA2_ERR_INVALID_ARG


def test_varlen_empty_batch_launches_nothing(lib):
    before = lib.fa2_kernel_launches()
    assert call_fwd_varlen(lib, total=0, q=None, k=None, v=None, o=None, lse=None) == F.FA2_OK
    assert lib.fa2_kernel_launches() == before


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_varlen_call_without_device_is_cuda_error(lib):
    assert call_fwd_varlen(lib) == F.FA2_ERR_CUDA


def test_bwd_varlen_checks_its_workspace(lib):
    need = lib.fa2_bwd_workspace_size(1, 1000, 16, 128, F.FA2_BF16, 0)
    assert need == 1000 * 16 * 128 * 4
    args = [P, P, P, P, P, P, ctypes.c_void_p(0x300000), ctypes.c_void_p(0x400000),
            ctypes.c_void_p(0x500000), ctypes.c_void_p(0x600000), need - 1, CU, 3, 512, 1000,
            16, 128, F.FA2_BF16] + [SP] * 7 + [0.0, 0, -1, -1, None, 0.0, 0, 0, None]
    assert lib.fa2_bwd_varlen(*args) == F.FA2_ERR_INVALID_ARG
    args[11] = None                     # no cu_seqlens
    args[10] = need
    assert lib.fa2_bwd_varlen(*args) == F.FA2_ERR_INVALID_ARG


# ----------------------------------------------------------------- block-sparse
def call_fwd_bs(lib, **kw):
    a = dict(q=P, k=P, v=P, o=ctypes.c_void_p(0x200000), lse=P, mask=ctypes.c_void_p(0x800000),
             sb=0, sh=0, d=128, dropout=0.0)
    a.update(kw)
    return lib.fa2_fwd_blocksparse(a["q"], a["k"], a["v"], a["o"], a["lse"], 1, 256, 2, a["d"],
                                   F.FA2_BF16, S128, S128, S128, S128, a["mask"], a["sb"], a["sh"],
                                   0.0, 0, -1, -1, None, a["dropout"], 0, None)


@pytest.mark.parametrize("bad", [dict(mask=None), dict(sb=-1), dict(sh=-4), dict(d=80),
                                 dict(q=None), dict(o=P), dict(dropout=2.0)])
def test_fwd_blocksparse_rejects_invalid(lib, bad):
    assert call_fwd_bs(lib, **bad) == F.FA2_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_blocksparse_call_without_device_is_cuda_error(lib):
    assert call_fwd_bs(lib) == F.FA2_ERR_CUDA


# ----------------------------------------------------------------- e4m3 forward
S8 = F.Strides(2048 * 16 * 128, 16 * 128, 128)   # e4m3 [B, N, H=16, 128] (bytes)


def call_fwd_fp8(lib, **kw):
    a = dict(q=P, o=ctypes.c_void_p(0x200000), d=128, sq=S8, qd=1.0)
    a.update(kw)
    return lib.fa2_fwd_fp8(a["q"], P, P, a["o"], P, 1, 256, 16, a["d"], a["sq"], S8, S8, S128,
                           a["qd"], 1.0, 1.0, 0.0, 0, -1, -1, None, None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(o=P), dict(qd=0.0), dict(qd=float("inf")),
                                 dict(qd=float("nan")), dict(sq=F.Strides(8, 16 * 128, 128)),
                                 dict(d=100)])
def test_fwd_fp8_rejects_invalid(lib, bad):
    assert call_fwd_fp8(lib, **bad) == F.FA2_ERR_INVALID_ARG


def test_fwd_fp8_head_dim_64_unsupported(lib):
    assert call_fwd_fp8(lib, d=64, sq=F.Strides(2048 * 16 * 64, 16 * 64, 64)) == \
        F.FA2_ERR_UNSUPPORTED
