"""Exact FlashAttention-2 (forward + backward) for NVIDIA B200, sm_100a.

The compute path is libfa2.so (CUDA kernels behind the C ABI in
include/fa2.h); ``exact_attention_147_b200.fa2`` is its Python binding.
"""

from .fa2 import (  # noqa: F401
    bwd,
    bwd_preprocess,
    device_status,
    flash_attention_v2,
    fwd,
    load_library,
    set_wait_limit_ms,
    workspace_size,
)
