"""ctypes binding of include/moe_q2.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_q2.so")

MOE_OK = 0
_lib = None


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {moe_status_str(code)} (status {code})")
        self.code = code


class moe_dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32)]


class moe_router(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


class moe_experts(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p)]


class moe_shared(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p)]


EXPORTED = [
    "moe_canonical_expert_bytes",
    "moe_packed_expert_bytes",
    "moe_pack_q2",
    "moe_workspace_bytes",
    "moe_route",
    "moe_route_noalloc",
    "moe_layer_forward",
    "moe_layer_forward_host",
    "moe_layer_forward_residual",
    "moe_experts_forward",
    "moe_dispatch",
    "moe_rmsnorm_residual",
    "moe_trace_kernel",
    "moe_set_cold_expert_tokens",
    "moe_check_status",
    "moe_status_str",
]


def lib():
    """Load libmoe_q2.so (built by bit_block_quantized_moe_b200.build); fails loudly if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing (run __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        D = ctypes.POINTER(moe_dims)
        L.moe_canonical_expert_bytes.restype = sz
        L.moe_canonical_expert_bytes.argtypes = [D]
        L.moe_packed_expert_bytes.restype = sz
        L.moe_packed_expert_bytes.argtypes = [D]
        L.moe_pack_q2.restype = ctypes.c_int
        L.moe_pack_q2.argtypes = [D, P, i32, P, sz, P]
        L.moe_workspace_bytes.restype = sz
        L.moe_workspace_bytes.argtypes = [D, i32]
        L.moe_route.restype = ctypes.c_int
        L.moe_route.argtypes = [D, P, ctypes.POINTER(moe_router), i32, P, P, P, sz, P]
        L.moe_route_noalloc.restype = ctypes.c_int
        L.moe_route_noalloc.argtypes = [D, P, ctypes.POINTER(moe_router), i32, P, P, P]
        L.moe_layer_forward.restype = ctypes.c_int
        L.moe_layer_forward.argtypes = [D, P, ctypes.POINTER(moe_router), ctypes.POINTER(moe_experts),
                                        ctypes.POINTER(moe_shared), P, i32, P, P, P, sz, P]
        L.moe_layer_forward_host.restype = ctypes.c_int
        L.moe_layer_forward_host.argtypes = [D, P, ctypes.POINTER(moe_router), ctypes.POINTER(moe_experts),
                                             ctypes.POINTER(moe_shared), P, i32, P, P, P, sz, P]
        L.moe_layer_forward_residual.restype = ctypes.c_int
        L.moe_layer_forward_residual.argtypes = [D, P, ctypes.POINTER(moe_router), ctypes.POINTER(moe_experts),
                                                 ctypes.POINTER(moe_shared), P, P, ctypes.c_float, i32, P, P, P, sz,
                                                 P]
        L.moe_experts_forward.restype = ctypes.c_int
        L.moe_experts_forward.argtypes = [D, P, P, P, ctypes.POINTER(moe_experts), ctypes.POINTER(moe_shared), P,
                                          i32, P, sz, P]
        L.moe_dispatch.restype = ctypes.c_int
        L.moe_dispatch.argtypes = [D, P, i32, P, P, P, P, P, sz, P]
        L.moe_rmsnorm_residual.restype = ctypes.c_int
        L.moe_rmsnorm_residual.argtypes = [P, P, P, i32, i32, ctypes.c_float, P]
        L.moe_trace_kernel.restype = ctypes.c_int
        L.moe_trace_kernel.argtypes = [i32, P, P]
        L.moe_set_cold_expert_tokens.restype = ctypes.c_int
        L.moe_set_cold_expert_tokens.argtypes = [i32]
        L.moe_check_status.restype = ctypes.c_int
        L.moe_check_status.argtypes = [P, P]
        L.moe_status_str.restype = ctypes.c_char_p
        L.moe_status_str.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int, what: str):
    if code != MOE_OK:
        raise MoeError(code, what)


def _dims(d) -> moe_dims:
    if isinstance(d, moe_dims):
        return d
    return moe_dims(int(d[0]), int(d[1]), int(d[2]), int(d[3]))


def moe_status_str(code: int) -> str:
    return lib().moe_status_str(int(code)).decode()


def moe_canonical_expert_bytes(dims) -> int:
    return int(lib().moe_canonical_expert_bytes(ctypes.byref(_dims(dims))))


def moe_packed_expert_bytes(dims) -> int:
    return int(lib().moe_packed_expert_bytes(ctypes.byref(_dims(dims))))


def moe_workspace_bytes(dims, max_T: int) -> int:
    return int(lib().moe_workspace_bytes(ctypes.byref(_dims(dims)), int(max_T)))


def moe_pack_q2(dims, canonical, n_experts: int, packed, stream=None):
    code = lib().moe_pack_q2(ctypes.byref(_dims(dims)), _ptr(canonical), int(n_experts), _ptr(packed),
                             packed.numel() * packed.element_size(), _stream(stream))
    _check(code, "moe_pack_q2")


def moe_route(dims, x, router_w, router_b, T: int, topk_idx, topk_w, workspace, stream=None):
    r = moe_router(_ptr(router_w), _ptr(router_b))
    code = lib().moe_route(ctypes.byref(_dims(dims)), _ptr(x), ctypes.byref(r), int(T), _ptr(topk_idx),
                           _ptr(topk_w), _ptr(workspace), workspace.numel() * workspace.element_size(),
                           _stream(stream))
    _check(code, "moe_route")


def moe_route_noalloc(dims, x, router_w, router_b, T: int, topk_idx, topk_w, stream=None):
    """moe_route without a workspace: the library's own static device scratch holds the
    logits, for callers that cannot allocate device memory (see include/moe_q2.h)."""
    r = moe_router(_ptr(router_w), _ptr(router_b))
    code = lib().moe_route_noalloc(ctypes.byref(_dims(dims)), _ptr(x), ctypes.byref(r), int(T), _ptr(topk_idx),
                                   _ptr(topk_w), _stream(stream))
    _check(code, "moe_route_noalloc")


def moe_layer_forward(dims, x, router_w, router_b, experts_packed, shared_packed, out, T: int, workspace,
                      topk_idx_out=None, topk_w_out=None, stream=None):
    r = moe_router(_ptr(router_w), _ptr(router_b))
    ex = moe_experts(_ptr(experts_packed))
    sh = moe_shared(_ptr(shared_packed))
    code = lib().moe_layer_forward(ctypes.byref(_dims(dims)), _ptr(x), ctypes.byref(r), ctypes.byref(ex),
                                   ctypes.byref(sh), _ptr(out), int(T), _ptr(topk_idx_out), _ptr(topk_w_out),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "moe_layer_forward")


def moe_layer_forward_host(dims, x_host, router_w, router_b, experts_packed, shared_packed, out_host, T: int,
                           workspace, topk_idx_out=None, topk_w_out=None, stream=None):
    """x_host / out_host: page-locked host tensors (e.g. torch's pin_memory()), T <= 8."""
    r = moe_router(_ptr(router_w), _ptr(router_b))
    ex = moe_experts(_ptr(experts_packed))
    sh = moe_shared(_ptr(shared_packed))
    code = lib().moe_layer_forward_host(ctypes.byref(_dims(dims)), _ptr(x_host), ctypes.byref(r), ctypes.byref(ex),
                                        ctypes.byref(sh), _ptr(out_host), int(T), _ptr(topk_idx_out),
                                        _ptr(topk_w_out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream))
    _check(code, "moe_layer_forward_host")


def moe_layer_forward_residual(dims, x_norm_in, router_w, router_b, experts_packed, shared_packed, resid, x_norm_out,
                               T: int, workspace, eps: float = 1e-6, topk_idx_out=None, topk_w_out=None,
                               stream=None):
    r = moe_router(_ptr(router_w), _ptr(router_b))
    ex = moe_experts(_ptr(experts_packed))
    sh = moe_shared(_ptr(shared_packed))
    code = lib().moe_layer_forward_residual(ctypes.byref(_dims(dims)), _ptr(x_norm_in), ctypes.byref(r),
                                            ctypes.byref(ex), ctypes.byref(sh), _ptr(resid), _ptr(x_norm_out),
                                            float(eps), int(T), _ptr(topk_idx_out), _ptr(topk_w_out),
                                            _ptr(workspace), workspace.numel() * workspace.element_size(),
                                            _stream(stream))
    _check(code, "moe_layer_forward_residual")


def moe_experts_forward(dims, x, topk_idx, topk_w, experts_packed, shared_packed, out, T: int, workspace,
                        stream=None):
    ex = moe_experts(_ptr(experts_packed))
    sh = moe_shared(_ptr(shared_packed))
    code = lib().moe_experts_forward(ctypes.byref(_dims(dims)), _ptr(x), _ptr(topk_idx), _ptr(topk_w),
                                     ctypes.byref(ex), ctypes.byref(sh), _ptr(out), int(T), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "moe_experts_forward")


def moe_dispatch(dims, topk_idx, T: int, counts, offsets, perm, inv, workspace, stream=None):
    code = lib().moe_dispatch(ctypes.byref(_dims(dims)), _ptr(topk_idx), int(T), _ptr(counts), _ptr(offsets),
                              _ptr(perm), _ptr(inv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream))
    _check(code, "moe_dispatch")


def moe_rmsnorm_residual(resid, y, x_norm, T: int, hidden: int, eps: float = 1e-6, stream=None):
    code = lib().moe_rmsnorm_residual(_ptr(resid), _ptr(y), _ptr(x_norm), int(T), int(hidden), float(eps),
                                      _stream(stream))
    _check(code, "moe_rmsnorm_residual")


MOE_KERNEL = {"router_logits": 0, "topk": 1, "dispatch_bits": 2, "dispatch_scan": 3, "dispatch_place": 4,
              "gate_up": 5, "down": 6, "combine": 7, "decode_fused": 8,
              "gather": 9}


def moe_trace_kernel(kernel_id: int, before=None, after=None):
    """Record torch.cuda.Event `before`/`after` (created with external=True) around kernel `kernel_id`."""
    b = None if before is None else before.cuda_event
    a = None if after is None else after.cuda_event
    _check(lib().moe_trace_kernel(int(kernel_id), b, a), "moe_trace_kernel")


def moe_set_cold_expert_tokens(max_tokens: int):
    """Per host thread: in a prefill chunk, experts with at most max_tokens tokens run on the register-dequant
    kernels (0, the default: every expert on the tcgen05 kernels)."""
    _check(lib().moe_set_cold_expert_tokens(int(max_tokens)), "moe_set_cold_expert_tokens")


def moe_check_status(workspace, stream=None):
    code = lib().moe_check_status(_ptr(workspace), _stream(stream))
    _check(code, "moe_check_status")
