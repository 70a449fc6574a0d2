"""Python binding of libfa2 (argument marshalling only).

Every step of the attention computation runs in libfa2's CUDA kernels; this
module only allocates outputs with PyTorch, reads strides and the current
CUDA stream, and calls the C ABI of ``include/fa2.h`` through ctypes.  If
the shared library is missing it raises -- there is no other code path.

The user-facing call mirrors the one printed in the "FlashAttention v2"
article (wmrh.cn), §5.1::

    flash_attention_v2(q, k, v, dropout_p=0.0, softmax_scale=None,
                       causal=False, window_size=(-1, -1),
                       alibi_slopes=None, deterministic=False)

with q, k, v laid out as [batch, seqlen, heads, head_dim].
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa2.so")

FA2_BF16 = 0
FA2_F32 = 1
FA2_OK = 0
FA2_ERR_INVALID_ARG = 1
FA2_ERR_UNSUPPORTED = 2
FA2_ERR_CUDA = 3
FA2_ERR_DEVICE_TIMEOUT = 4
FA2_ERR_SCRATCH_LIMIT = 5
NOALLOC_MAX_DQ_FLOATS = 4 * 1024 * 1024

# Every symbol include/fa2.h declares.
EXPORTED = ("fa2_fwd", "fa2_bwd_preprocess", "fa2_bwd_workspace_size", "fa2_bwd",
            "fa2_fwd_varlen", "fa2_bwd_varlen", "fa2_fwd_blocksparse", "fa2_bwd_blocksparse",
            "fa2_fwd_fp8",
            "fa2_strerror", "fa2_device_status",
            "fa2_set_wait_limit_ms", "fa2_kernel_launches", "fa2_bwd_noalloc",
            "fa2_test_skip_arrive")
# Device status code of a packed call whose cu_seqlens was malformed.
STATUS_BAD_SEQLENS = 0xF10


class Strides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("n", ctypes.c_int64), ("h", ctypes.c_int64)]


class Fa2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {strerror(status)} (status {status})")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libfa2.so and declare its signatures (raises if it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libfa2.so not found at {path}; build it with "
            "`python -m exact_attention_147_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, s = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, Strides
    u64 = ctypes.c_uint64
    lib.fa2_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, s, s, s, s, f, i, i, i, vp, f, u64, vp]
    lib.fa2_fwd.restype = i
    lib.fa2_bwd_preprocess.argtypes = [vp, vp, vp, i, i, i, i, i, s, s, vp]
    lib.fa2_bwd_preprocess.restype = i
    lib.fa2_bwd_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.fa2_bwd_workspace_size.restype = ctypes.c_size_t
    lib.fa2_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                            i, i, i, i, i, s, s, s, s, s, s, s, f, i, i, i, vp, f, u64, i, vp]
    lib.fa2_bwd.restype = i
    lib.fa2_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, s, s, s, s, f, i, i, i,
                                   vp, f, u64, vp]
    lib.fa2_fwd_varlen.restype = i
    lib.fa2_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp,
                                   i, i, i, i, i, i, s, s, s, s, s, s, s, f, i, i, i, vp, f, u64,
                                   i, vp]
    lib.fa2_bwd_varlen.restype = i
    i64 = ctypes.c_int64
    lib.fa2_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, s, s, s, s, vp, i64, i64,
                                        f, i, i, i, vp, f, u64, vp]
    lib.fa2_fwd_blocksparse.restype = i
    lib.fa2_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                        i, i, i, i, i, s, s, s, s, s, s, s, vp, i64, i64, f, i, i, i,
                                        vp, f, u64, i, vp]
    lib.fa2_bwd_blocksparse.restype = i
    lib.fa2_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, s, s, s, s, f, f, f, f, i, i, i, vp,
                                vp]
    lib.fa2_fwd_fp8.restype = i
    lib.fa2_strerror.argtypes = [i]
    lib.fa2_strerror.restype = ctypes.c_char_p
    lib.fa2_device_status.argtypes = [ctypes.POINTER(ctypes.c_int), i]
    lib.fa2_device_status.restype = i
    lib.fa2_set_wait_limit_ms.argtypes = [i]
    lib.fa2_set_wait_limit_ms.restype = i
    lib.fa2_test_skip_arrive.argtypes = [i]
    lib.fa2_test_skip_arrive.restype = i
    lib.fa2_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i,
                                    s, s, s, s, s, s, s, f, i, i, i, vp, f, vp]
    lib.fa2_bwd_noalloc.restype = i
    lib.fa2_kernel_launches.argtypes = []
    lib.fa2_kernel_launches.restype = ctypes.c_uint64
    _lib = lib
    return lib


def strerror(status: int) -> str:
    return load_library().fa2_strerror(int(status)).decode()


def _check(status: int, what: str):
    if status != FA2_OK:
        raise Fa2Error(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FA2_BF16
    if t.dtype == torch.float32:
        return FA2_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _strides(t: torch.Tensor) -> Strides:
    if t.dim() != 4:
        raise ValueError("expected a [batch, seqlen, heads, head_dim] tensor")
    if t.stride(3) != 1:
        raise ValueError("head_dim must be contiguous (stride 1)")
    return Strides(t.stride(0), t.stride(1), t.stride(2))


def _packed_strides(t: torch.Tensor) -> Strides:
    if t.dim() != 3:
        raise ValueError("expected a packed [total, heads, head_dim] tensor")
    if t.stride(2) != 1:
        raise ValueError("head_dim must be contiguous (stride 1)")
    return Strides(0, t.stride(0), t.stride(1))


def _seqlens(cu_seqlens: torch.Tensor) -> torch.Tensor:
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor of B + 1 offsets")
    return cu_seqlens.contiguous()


BLOCK = 128  # side of a block-mask block


def _block_mask(block_mask: torch.Tensor, B: int, H: int, N: int):
    """(tensor, batch stride, head stride) of a [B, H, nb, nb] uint8 block mask
    (batch and head strides may be 0: one mask shared)."""
    nb = (N + BLOCK - 1) // BLOCK
    if block_mask.dtype not in (torch.uint8, torch.bool) or block_mask.dim() != 4:
        raise ValueError("block_mask must be a [B, H, nb, nb] uint8 or bool tensor")
    if tuple(block_mask.shape) != (B, H, nb, nb):
        raise ValueError(f"block_mask shape {tuple(block_mask.shape)} != {(B, H, nb, nb)}")
    m = block_mask.view(torch.uint8) if block_mask.dtype == torch.bool else block_mask
    if m.stride(3) != 1 or m.stride(2) != nb:
        m = m.contiguous()
    return m, m.stride(0), m.stride(1)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _window(causal, window_size):
    wl, wr = window_size if window_size is not None else (-1, -1)
    return int(bool(causal)), int(wl), int(wr)


def _scale(softmax_scale):
    return 0.0 if softmax_scale is None else float(softmax_scale)


def fwd(q, k, v, softmax_scale=None, causal=False, window_size=(-1, -1),
        alibi_slopes=None, dropout_p=0.0, out=None, lse=None, stream=None, dropout_seed=0):
    """Forward pass; returns (out [B,N,H,d], lse [B,H,N] fp32)."""
    lib = load_library()
    B, N, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    c, wl, wr = _window(causal, window_size)
    st = lib.fa2_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, N, H, d,
                     _dtype_code(q), _strides(q), _strides(k), _strides(v), _strides(out),
                     _scale(softmax_scale), c, wl, wr, _ptr(alibi_slopes),
                     float(dropout_p), int(dropout_seed) & 0xFFFFFFFFFFFFFFFF, _stream(stream))
    _check(st, "fa2_fwd")
    return out, lse


def bwd_preprocess(out, dout, D=None, stream=None):
    """D[b,h,i] = sum_c dout[b,i,h,c] * out[b,i,h,c] (fp32).

    Packed [total, H, d] tensors give D as [H, total]."""
    if out.dim() == 3:
        total, H, _ = out.shape
        if D is None:
            D = torch.empty((H, total), dtype=torch.float32, device=out.device)
        if total > 0:
            bwd_preprocess(out.unsqueeze(0), dout.unsqueeze(0), D.unsqueeze(0), stream)
        return D
    lib = load_library()
    B, N, H, d = out.shape
    if D is None:
        D = torch.empty((B, H, N), dtype=torch.float32, device=out.device)
    st = lib.fa2_bwd_preprocess(_ptr(out), _ptr(dout), _ptr(D), B, N, H, d, _dtype_code(out),
                                _strides(out), _strides(dout), _stream(stream))
    _check(st, "fa2_bwd_preprocess")
    return D


def workspace_size(B, N, H, d, dtype, deterministic=False) -> int:
    code = FA2_BF16 if dtype == torch.bfloat16 else FA2_F32
    return int(load_library().fa2_bwd_workspace_size(B, N, H, d, code, int(bool(deterministic))))


def bwd(dout, q, k, v, lse, D, softmax_scale=None, causal=False, window_size=(-1, -1),
        alibi_slopes=None, dropout_p=0.0, deterministic=False, dq=None, dk=None, dv=None,
        workspace=None, stream=None, dropout_seed=0):
    """Backward pass; returns (dq, dk, dv) shaped like q, k, v."""
    lib = load_library()
    B, N, H, d = q.shape
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = workspace_size(B, N, H, d, q.dtype, deterministic)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    c, wl, wr = _window(causal, window_size)
    st = lib.fa2_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lse), _ptr(D), _ptr(dq),
                     _ptr(dk), _ptr(dv), _ptr(workspace), wbytes, B, N, H, d, _dtype_code(q),
                     _strides(q), _strides(k), _strides(v), _strides(dout), _strides(dq),
                     _strides(dk), _strides(dv), _scale(softmax_scale), c, wl, wr,
                     _ptr(alibi_slopes), float(dropout_p),
                     int(dropout_seed) & 0xFFFFFFFFFFFFFFFF, int(bool(deterministic)),
                     _stream(stream))
    _check(st, "fa2_bwd")
    return dq, dk, dv


def fwd_varlen(q, k, v, cu_seqlens, max_seqlen, softmax_scale=None, causal=False,
               window_size=(-1, -1), alibi_slopes=None, dropout_p=0.0, out=None, lse=None,
               stream=None, dropout_seed=0):
    """Forward pass of a packed batch: q, k, v are [total, H, d], sequence b
    owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1 (int32, on the device).
    Returns (out [total, H, d], lse [H, total] fp32)."""
    lib = load_library()
    total, H, d = q.shape
    cu = _seqlens(cu_seqlens)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, total), dtype=torch.float32, device=q.device)
    c, wl, wr = _window(causal, window_size)
    st = lib.fa2_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu),
                            cu.numel() - 1, int(max_seqlen), total, H, d, _dtype_code(q),
                            _packed_strides(q), _packed_strides(k), _packed_strides(v),
                            _packed_strides(out), _scale(softmax_scale), c, wl, wr,
                            _ptr(alibi_slopes), float(dropout_p),
                            int(dropout_seed) & 0xFFFFFFFFFFFFFFFF, _stream(stream))
    _check(st, "fa2_fwd_varlen")
    return out, lse


def bwd_varlen(dout, q, k, v, lse, D, cu_seqlens, max_seqlen, softmax_scale=None,
               causal=False, window_size=(-1, -1), alibi_slopes=None, dropout_p=0.0,
               deterministic=False, dq=None, dk=None, dv=None, workspace=None, stream=None,
               dropout_seed=0):
    """Backward pass of a packed batch; returns (dq, dk, dv) shaped like q, k, v."""
    lib = load_library()
    total, H, d = q.shape
    cu = _seqlens(cu_seqlens)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = workspace_size(1, total, H, d, q.dtype, deterministic) if total > 0 else 0
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    c, wl, wr = _window(causal, window_size)
    st = lib.fa2_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lse), _ptr(D), _ptr(dq),
                            _ptr(dk), _ptr(dv), _ptr(workspace), wbytes, _ptr(cu),
                            cu.numel() - 1, int(max_seqlen), total, H, d, _dtype_code(q),
                            _packed_strides(q), _packed_strides(k), _packed_strides(v),
                            _packed_strides(dout), _packed_strides(dq), _packed_strides(dk),
                            _packed_strides(dv), _scale(softmax_scale), c, wl, wr,
                            _ptr(alibi_slopes), float(dropout_p),
                            int(dropout_seed) & 0xFFFFFFFFFFFFFFFF, int(bool(deterministic)),
                            _stream(stream))
    _check(st, "fa2_bwd_varlen")
    return dq, dk, dv


def fwd_blocksparse(q, k, v, block_mask, softmax_scale=None, causal=False,
                    window_size=(-1, -1), alibi_slopes=None, dropout_p=0.0, out=None, lse=None,
                    stream=None, dropout_seed=0):
    """Forward pass with a [B, H, ceil(N/128), ceil(N/128)] block mask (uint8
    or bool; nonzero = the 128 x 128 block may be attended)."""
    lib = load_library()
    B, N, H, d = q.shape
    m, msb, msh = _block_mask(block_mask, B, H, N)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    c, wl, wr = _window(causal, window_size)
    st = lib.fa2_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, N, H, d,
                                 _dtype_code(q), _strides(q), _strides(k), _strides(v),
                                 _strides(out), _ptr(m), msb, msh, _scale(softmax_scale), c, wl,
                                 wr, _ptr(alibi_slopes), float(dropout_p),
                                 int(dropout_seed) & 0xFFFFFFFFFFFFFFFF, _stream(stream))
    _check(st, "fa2_fwd_blocksparse")
    return out, lse


def bwd_blocksparse(dout, q, k, v, lse, D, block_mask, softmax_scale=None, causal=False,
                    window_size=(-1, -1), alibi_slopes=None, dropout_p=0.0, deterministic=False,
                    dq=None, dk=None, dv=None, workspace=None, stream=None, dropout_seed=0):
    """Backward pass with the forward's block mask; returns (dq, dk, dv)."""
    lib = load_library()
    B, N, H, d = q.shape
    m, msb, msh = _block_mask(block_mask, B, H, N)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = workspace_size(B, N, H, d, q.dtype, deterministic)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    c, wl, wr = _window(causal, window_size)
    st = lib.fa2_bwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lse), _ptr(D),
                                 _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), wbytes, B, N, H, d,
                                 _dtype_code(q), _strides(q), _strides(k), _strides(v),
                                 _strides(dout), _strides(dq), _strides(dk), _strides(dv),
                                 _ptr(m), msb, msh, _scale(softmax_scale), c, wl, wr,
                                 _ptr(alibi_slopes), float(dropout_p),
                                 int(dropout_seed) & 0xFFFFFFFFFFFFFFFF, int(bool(deterministic)),
                                 _stream(stream))
    _check(st, "fa2_bwd_blocksparse")
    return dq, dk, dv


def fwd_fp8(q, k, v, q_descale, k_descale, v_descale, softmax_scale=None, causal=False,
            window_size=(-1, -1), alibi_slopes=None, out=None, lse=None, stream=None):
    """Forward pass on e4m3 inputs (torch.float8_e4m3fn, [B, N, H, 128]) with
    per-tensor dequantisation factors; returns (out bf16, lse fp32)."""
    lib = load_library()
    for t in (q, k, v):
        if t.dtype != torch.float8_e4m3fn:
            raise TypeError("fwd_fp8 takes torch.float8_e4m3fn tensors")
    B, N, H, d = q.shape
    if out is None:
        out = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    c, wl, wr = _window(causal, window_size)
    st = lib.fa2_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, N, H, d, _strides(q),
                         _strides(k), _strides(v), _strides(out), float(q_descale),
                         float(k_descale), float(v_descale), _scale(softmax_scale), c, wl, wr,
                         _ptr(alibi_slopes), _stream(stream))
    _check(st, "fa2_fwd_fp8")
    return out, lse


def device_status(clear=True) -> int:
    """Device status word (0 = no kernel gave up a bounded wait)."""
    code = ctypes.c_int(0)
    st = load_library().fa2_device_status(ctypes.byref(code), int(bool(clear)))
    if st not in (FA2_OK, FA2_ERR_DEVICE_TIMEOUT):
        _check(st, "fa2_device_status")
    return int(code.value)


def kernel_launches() -> int:
    """Kernels launched by libfa2 in this process so far."""
    return int(load_library().fa2_kernel_launches())


def set_wait_limit_ms(ms: int):
    _check(load_library().fa2_set_wait_limit_ms(int(ms)), "fa2_set_wait_limit_ms")


def test_skip_arrive(which: int):
    """Test switch of the bounded-wait path: 1 = forward, 2 = backward, 0 = off
    (see fa2_test_skip_arrive in include/fa2.h)."""
    _check(load_library().fa2_test_skip_arrive(int(which)), "fa2_test_skip_arrive")


class _Fa2Function(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, dropout_p, softmax_scale, causal, window_size, alibi_slopes,
                deterministic):
        # a fresh mask per call, drawn from torch's default CPU generator
        seed = int(torch.randint(0, 2**63 - 1, (1,)).item()) if dropout_p > 0 else 0
        out, lse = fwd(q, k, v, softmax_scale, causal, window_size, alibi_slopes, dropout_p,
                       dropout_seed=seed)
        ctx.save_for_backward(q, k, v, out, lse, alibi_slopes)
        ctx.opts = (dropout_p, softmax_scale, causal, window_size, deterministic, seed)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse, alibi_slopes = ctx.saved_tensors
        dropout_p, softmax_scale, causal, window_size, deterministic, seed = ctx.opts
        dout = dout if dout.stride(-1) == 1 else dout.contiguous()
        D = bwd_preprocess(out, dout)
        dq, dk, dv = bwd(dout, q, k, v, lse, D, softmax_scale, causal, window_size,
                         alibi_slopes, dropout_p, deterministic, dropout_seed=seed)
        return dq, dk, dv, None, None, None, None, None, None


def flash_attention_v2(q, k, v, dropout_p=0.0, softmax_scale=None, causal=False,
                       window_size=(-1, -1), alibi_slopes=None, deterministic=False):
    """Exact attention with autograd support; q, k, v are [B, N, H, d]."""
    return _Fa2Function.apply(q, k, v, dropout_p, softmax_scale, causal, window_size,
                              alibi_slopes, deterministic)


class _Fa2VarlenFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, cu_seqlens, max_seqlen, dropout_p, softmax_scale, causal,
                window_size, alibi_slopes, deterministic):
        seed = int(torch.randint(0, 2**63 - 1, (1,)).item()) if dropout_p > 0 else 0
        out, lse = fwd_varlen(q, k, v, cu_seqlens, max_seqlen, softmax_scale, causal,
                              window_size, alibi_slopes, dropout_p, dropout_seed=seed)
        ctx.save_for_backward(q, k, v, out, lse, cu_seqlens, alibi_slopes)
        ctx.opts = (max_seqlen, dropout_p, softmax_scale, causal, window_size, deterministic,
                    seed)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse, cu_seqlens, alibi_slopes = ctx.saved_tensors
        max_seqlen, dropout_p, softmax_scale, causal, window_size, deterministic, seed = ctx.opts
        dout = dout if dout.stride(-1) == 1 else dout.contiguous()
        D = bwd_preprocess(out, dout)
        dq, dk, dv = bwd_varlen(dout, q, k, v, lse, D, cu_seqlens, max_seqlen, softmax_scale,
                                causal, window_size, alibi_slopes, dropout_p, deterministic,
                                dropout_seed=seed)
        return dq, dk, dv, None, None, None, None, None, None, None, None


def flash_attention_v2_varlen(q, k, v, cu_seqlens, max_seqlen, dropout_p=0.0,
                              softmax_scale=None, causal=False, window_size=(-1, -1),
                              alibi_slopes=None, deterministic=False):
    """Exact attention of a packed batch with autograd support: q, k, v are
    [total, H, d] and sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1."""
    return _Fa2VarlenFunction.apply(q, k, v, cu_seqlens, max_seqlen, dropout_p, softmax_scale,
                                    causal, window_size, alibi_slopes, deterministic)


class _Fa2BlockSparseFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, block_mask, dropout_p, softmax_scale, causal, window_size,
                alibi_slopes, deterministic):
        seed = int(torch.randint(0, 2**63 - 1, (1,)).item()) if dropout_p > 0 else 0
        out, lse = fwd_blocksparse(q, k, v, block_mask, softmax_scale, causal, window_size,
                                   alibi_slopes, dropout_p, dropout_seed=seed)
        ctx.save_for_backward(q, k, v, out, lse, block_mask, alibi_slopes)
        ctx.opts = (dropout_p, softmax_scale, causal, window_size, deterministic, seed)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse, block_mask, alibi_slopes = ctx.saved_tensors
        dropout_p, softmax_scale, causal, window_size, deterministic, seed = ctx.opts
        dout = dout if dout.stride(-1) == 1 else dout.contiguous()
        D = bwd_preprocess(out, dout)
        dq, dk, dv = bwd_blocksparse(dout, q, k, v, lse, D, block_mask, softmax_scale, causal,
                                     window_size, alibi_slopes, dropout_p, deterministic,
                                     dropout_seed=seed)
        return dq, dk, dv, None, None, None, None, None, None, None


def flash_attention_v2_blocksparse(q, k, v, block_mask, dropout_p=0.0, softmax_scale=None,
                                   causal=False, window_size=(-1, -1), alibi_slopes=None,
                                   deterministic=False):
    """Exact attention restricted to the 128 x 128 blocks a [B, H, nb, nb]
    block mask keeps, with autograd support; q, k, v are [B, N, H, d]."""
    return _Fa2BlockSparseFunction.apply(q, k, v, block_mask, dropout_p, softmax_scale, causal,
                                         window_size, alibi_slopes, deterministic)
