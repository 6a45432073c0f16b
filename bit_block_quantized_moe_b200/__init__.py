"""B200 (sm_100a) routed MoE layer over 2-bit block-quantized experts.

Python binding of the C ABI declared in ``include/moe_q2.h``: every function
here marshals torch tensors (CUDA ones, or page-locked host ones for
``moe_layer_forward_host``) into pointers and calls the function of the
same name in ``libmoe_q2.so``; all computation runs in that library's CUDA
kernels.  There is no fallback: if the library is missing, loading fails.
"""
from .binding import (  # noqa: F401
    MoeError,
    MOE_OK,
    lib,
    moe_canonical_expert_bytes,
    moe_check_status,
    moe_dims,
    moe_dispatch,
    moe_experts_forward,
    moe_layer_forward,
    moe_layer_forward_host,
    moe_layer_forward_residual,
    moe_pack_q2,
    moe_packed_expert_bytes,
    moe_rmsnorm_residual,
    moe_route,
    moe_route_noalloc,
    moe_set_cold_expert_tokens,
    moe_status_str,
    moe_trace_kernel,
    MOE_KERNEL,
    moe_workspace_bytes,
)
from .layer import Q2MoeLayer  # noqa: F401
