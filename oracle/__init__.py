"""fp64 CPU parity oracle for the routed MoE layer over Q2 block-quantized experts.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the bench's CPU-baseline leg may import this package.  It shares no code with
the CUDA library: the arithmetic lives in ``oracle_moe.c`` (plain C, binary64,
OpenMP over independent tokens), compiled here with gcc and called through
ctypes.  Inputs come from the seeded generator in ``gen``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle_moe.c")
_HDR = os.path.join(_HERE, "oracle_moe.h")
_OUT_DIR = os.path.join(_HERE, "_build")
_SO = os.path.join(_OUT_DIR, "liboracle_moe.so")
_lib = None

QBLOCK = 32
QBLOCK_BYTES = 10


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2, no fast-math, OpenMP) if missing or stale."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    stale = not os.path.exists(_SO) or max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)) > os.path.getmtime(_SO)
    if force or stale:
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.orc_half_to_double.restype = ctypes.c_double
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_double.restype = ctypes.c_double
        L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.orc_double_to_bf16.restype = ctypes.c_uint16
        L.orc_double_to_bf16.argtypes = [ctypes.c_double]
        L.orc_double_to_bf16_array.argtypes = [ctypes.c_size_t, P, P]
        L.orc_dequant_block.argtypes = [P, P]
        L.orc_dequant_matrix.argtypes = [P, i, i, P]
        L.orc_expert_bytes.restype = ctypes.c_size_t
        L.orc_expert_bytes.argtypes = [i, i]
        L.orc_silu.restype = ctypes.c_double
        L.orc_silu.argtypes = [ctypes.c_double]
        L.orc_expert_forward.argtypes = [i, i, P, P, P]
        L.orc_topk_one.argtypes = [P, i, i, P, P, P]
        L.orc_route.restype = i
        L.orc_route.argtypes = [i, i, i, i, P, P, P, P, P, P, P]
        L.orc_layer.restype = i
        L.orc_layer.argtypes = [i, i, i, i, i, P, P, P, P, P, P, P, P, P, P]
        L.orc_rmsnorm.argtypes = [i, P, ctypes.c_double, P]
        L.orc_stack.restype = i
        L.orc_stack.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, ctypes.c_double, P, ctypes.c_double, P, P, P,
                                ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        L.orc_num_threads.restype = i
        L.orc_set_num_threads.argtypes = [i]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Threads for the oracle's token loops (n < 1: all host threads)."""
    lib().orc_set_num_threads(int(n))


def half_to_double(bits: int) -> float:
    return float(lib().orc_half_to_double(int(bits)))


def bf16_to_double(bits: int) -> float:
    return float(lib().orc_bf16_to_double(int(bits)))


def double_to_bf16(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().orc_double_to_bf16_array(v.size, _p(v), _p(out))
    return out


def dequant_block(block: np.ndarray) -> np.ndarray:
    blk = _c(block, np.uint8)
    assert blk.size == QBLOCK_BYTES
    w = np.empty(QBLOCK, dtype=np.float64)
    lib().orc_dequant_block(_p(blk), _p(w))
    return w


def dequant_matrix(blocks: np.ndarray, rows: int, cols: int) -> np.ndarray:
    blk = _c(blocks, np.uint8)
    assert blk.size == rows * cols // QBLOCK * QBLOCK_BYTES
    W = np.empty((rows, cols), dtype=np.float64)
    lib().orc_dequant_matrix(_p(blk), rows, cols, _p(W))
    return W


def expert_bytes(hidden: int, inter: int) -> int:
    return int(lib().orc_expert_bytes(hidden, inter))


def silu(z: float) -> float:
    return float(lib().orc_silu(float(z)))


def expert_forward(hidden: int, inter: int, expert: np.ndarray, x: np.ndarray) -> np.ndarray:
    ex = _c(expert, np.uint8)
    xv = _c(x, np.float64)
    y = np.empty(hidden, dtype=np.float64)
    lib().orc_expert_forward(hidden, inter, _p(ex), _p(xv), _p(y))
    return y


def topk(logits: np.ndarray, top_k: int):
    """Top-k of a logit matrix [T, E] (fp64): (idx [T,k] int32, w [T,k], gap [T])."""
    lg = np.atleast_2d(_c(logits, np.float64))
    T, E = lg.shape
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float64)
    gap = np.empty(T, dtype=np.float64)
    for t in range(T):
        row = np.ascontiguousarray(lg[t])
        g = np.empty(1, dtype=np.float64)
        lib().orc_topk_one(_p(row), E, top_k, _p(idx[t]), _p(w[t]), _p(g))
        gap[t] = g[0]
    return idx, w, gap


def route(x_bits: np.ndarray, router_w: np.ndarray, router_b, top_k: int):
    """Router + top-k for bf16 tokens x [T, H]: (idx, w, gap, logits)."""
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    Wr = _c(router_w, np.float32)
    E = Wr.shape[0]
    b = _c(router_b, np.float32)
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float64)
    gap = np.empty(T, dtype=np.float64)
    logits = np.empty((T, E), dtype=np.float64)
    rc = lib().orc_route(H, E, top_k, T, _p(x), _p(Wr), _p(b), _p(idx), _p(w), _p(gap), _p(logits))
    if rc:
        raise ValueError("oracle route: bad dimensions")
    return idx, w, gap, logits


def layer(x_bits, router_w, router_b, experts, shared, top_k: int, inter: int, forced_idx=None):
    """The whole layer for bf16 tokens x [T, H]: (y [T,H] fp64, idx, w, gap)."""
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    Wr = _c(router_w, np.float32)
    E = Wr.shape[0]
    b = _c(router_b, np.float32)
    ex = _c(experts, np.uint8)
    sh = _c(shared, np.uint8)
    assert ex.size == E * expert_bytes(H, inter) and sh.size == expert_bytes(H, inter)
    fi = _c(forced_idx, np.int32)
    y = np.empty((T, H), dtype=np.float64)
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float64)
    gap = np.empty(T, dtype=np.float64)
    rc = lib().orc_layer(H, inter, E, top_k, T, _p(x), _p(Wr), _p(b), _p(ex), _p(sh), _p(fi), _p(y), _p(idx),
                         _p(w), _p(gap))
    if rc:
        raise ValueError("oracle layer: bad dimensions")
    return y, idx, w, gap


def rmsnorm(v: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    a = np.atleast_2d(_c(v, np.float64))
    out = np.empty_like(a)
    for r in range(a.shape[0]):
        row = np.ascontiguousarray(a[r])
        o = np.empty_like(row)
        lib().orc_rmsnorm(a.shape[1], _p(row), float(eps), _p(o))
        out[r] = o
    return out.reshape(np.shape(v))


def stack(x_bits, layers, top_k: int, inter: int, eps: float = 1e-6, follow_idx=None, tie_gap: float = 1e-5,
          resid_in=None):
    """A stack of layers over bf16 tokens x [T, H]: r_0 = x; r_{l+1} = r_l + layer_l(bf16(RMSNorm(r_l))),
    the residual in fp64.  ``layers`` is a list of dicts with router_w, router_b, experts, shared (as
    gen.make_layer returns).  ``follow_idx`` [L, T, k] (optional): a routing made elsewhere that the stack
    takes at near-ties (see orc_stack).  Returns (resid [T,H] fp64, idx [L,T,k], gap [L,T], n_followed,
    n_mismatch).  ``resid_in`` [T, H] fp64 (optional): start from this residual instead of x."""
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    L = len(layers)
    keep = []

    def arr(key, dtype):
        vals = [None if lay[key] is None else _c(lay[key], dtype) for lay in layers]
        keep.append(vals)
        return (ctypes.c_void_p * max(L, 1))(*[None if v is None else v.ctypes.data for v in vals])

    E = np.asarray(layers[0]["router_w"]).shape[0] if L else top_k  # no layers: nothing is routed
    for lay in layers:
        assert np.asarray(lay["experts"]).size == E * expert_bytes(H, inter)
    rw, ex, sh = arr("router_w", np.float32), arr("experts", np.uint8), arr("shared", np.uint8)
    rb = arr("router_b", np.float32) if L and all(lay["router_b"] is not None for lay in layers) else None
    fi = _c(follow_idx, np.int32)
    if fi is not None:
        assert fi.shape == (L, T, top_k)
    r_in = _c(resid_in, np.float64)
    if r_in is not None:
        assert r_in.shape == (T, H)
    resid = np.empty((T, H), dtype=np.float64)
    idx = np.empty((L, T, top_k), dtype=np.int32)
    gap = np.empty((L, T), dtype=np.float64)
    nf, nm = ctypes.c_int(0), ctypes.c_int(0)
    rc = lib().orc_stack(H, inter, E, top_k, L, T, _p(x), _p(r_in), rw, rb, ex, sh, float(eps), _p(fi), float(tie_gap),
                         _p(resid), _p(idx), _p(gap), ctypes.byref(nf), ctypes.byref(nm))
    if rc:
        raise ValueError("oracle stack: bad dimensions")
    return resid, idx, gap, nf.value, nm.value
