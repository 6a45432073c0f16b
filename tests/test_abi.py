"""The C-ABI library: it loads, exports every declared entry point, and its
host-side checks reject bad arguments before touching a device (no GPU needed)."""
import ctypes
import os
import re

import pytest

import __graft_entry__
from bit_block_quantized_moe_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    __graft_entry__.build()
    return B.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe_q2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(B.EXPORTED) == names


def test_sizes(lib):
    d = B.moe_dims(2048, 512, 512, 10)
    assert B.moe_canonical_expert_bytes(d) == 983040
    assert B.moe_packed_expert_bytes(d) == 983040
    assert B.moe_workspace_bytes(d, 1024) > B.moe_workspace_bytes(d, 3) > 0
    assert B.moe_workspace_bytes(d, -1) == 0


@pytest.mark.parametrize("dims", [(2048, 512, 512, 0), (2048, 512, 512, 33), (2000, 512, 512, 10),
                                  (2048, 500, 512, 10), (8192, 512, 512, 10), (256, 128, 4, 5),
                                  (256, 128, 65536, 10), (96, 128, 16, 2), (4224, 128, 16, 2), (256, 4224, 16, 2),
                                  (256, 160, 16, 2), (256, 128, 0, 1), (256, 128, 64, -1)])
def test_bad_dims_rejected(lib, dims):
    d = B.moe_dims(*dims)
    assert B.moe_packed_expert_bytes(d) == 0
    assert B.moe_workspace_bytes(d, 8) == 0
    r = B.moe_router(16, None)
    ex, sh = B.moe_experts(16), B.moe_shared(16)
    code = lib.moe_layer_forward(ctypes.byref(d), 16, ctypes.byref(r), ctypes.byref(ex), ctypes.byref(sh), 4096, 3,
                                 None, None, 16, 1 << 30, None)
    assert code == 1  # MOE_ERR_ARG


def test_host_checks_before_launch(lib):
    d = B.moe_dims(256, 128, 16, 2)
    ws = B.moe_workspace_bytes(d, 8)
    r = B.moe_router(0x1000, None)
    ex, sh = B.moe_experts(0x2000), B.moe_shared(0x3000)

    def call(x=0x4000, out=0x8000, T=8, wsp=0x10000, wsb=ws, rr=r):
        return lib.moe_layer_forward(ctypes.byref(d), x, ctypes.byref(rr), ctypes.byref(ex), ctypes.byref(sh), out,
                                     T, None, None, wsp, wsb, None)

    assert call(T=0) == 0                      # T = 0: no-op, nothing launched
    assert call(T=-1) == 1
    assert call(x=0x4001) == 2                 # misaligned x
    assert call(wsp=0x10008) == 2              # misaligned workspace
    assert call(wsb=ws - 1) == 3               # workspace too small
    assert call(out=0x4000 + 256) == 1         # out overlaps x
    assert call(rr=B.moe_router(None, None)) == 1
    assert lib.moe_check_status(None, None) == 1
    assert B.moe_status_str(3) == "workspace too small"
    assert lib.moe_pack_q2(ctypes.byref(d), 0x1000, -1, 0x2000, 1 << 20, None) == 1
    assert lib.moe_pack_q2(ctypes.byref(d), 0x1000, 0, 0x2000, 0, None) == 0
    assert lib.moe_pack_q2(ctypes.byref(d), 0x1000, 2, 0x2000, 100, None) == 1    # output too small
    assert lib.moe_pack_q2(ctypes.byref(d), 0x1000, 2, 0x2004, 1 << 20, None) == 2
    assert lib.moe_dispatch(ctypes.byref(d), 0x1000, 0, None, None, None, None, None, 0, None) == 0  # T = 0
    assert lib.moe_dispatch(ctypes.byref(d), 0x1000, 4, 0x2000, 0x3000, None, 0x5000, 0x10000, ws, None) == 1
    assert lib.moe_dispatch(ctypes.byref(d), 0x1000, 4, 0x2000, 0x3000, 0x4000, 0x5000, 0x10004, ws, None) == 2
    assert lib.moe_dispatch(ctypes.byref(d), 0x1000, 9, 0x2000, 0x3000, 0x4000, 0x5000, 0x10000, 16, None) == 3
    assert lib.moe_set_cold_expert_tokens(-1) == 1 and lib.moe_set_cold_expert_tokens(65) == 1
    assert lib.moe_set_cold_expert_tokens(8) == 0 and lib.moe_set_cold_expert_tokens(0) == 0
    assert lib.moe_rmsnorm_residual(None, None, None, 0, 256, 1e-6, None) == 0
    assert lib.moe_rmsnorm_residual(None, None, None, 4, 256, 1e-6, None) == 1


def test_host_memory_entry_point_checks(lib):
    """moe_layer_forward_host: the same argument checks as moe_layer_forward, and windows over 8 tokens refused,
    all before the device is touched (the host pointers here are never dereferenced)."""
    d = B.moe_dims(256, 128, 16, 2)
    r = B.moe_router(0x1000, None)
    ex, sh = B.moe_experts(0x2000), B.moe_shared(0x3000)

    def call(x=0x4000, out=0x8000, T=8, wsp=0x10000, wsb=None):
        wsb = B.moe_workspace_bytes(d, max(T, 1)) if wsb is None else wsb
        return lib.moe_layer_forward_host(ctypes.byref(d), x, ctypes.byref(r), ctypes.byref(ex), ctypes.byref(sh),
                                          out, T, None, None, wsp, wsb, None)

    assert call(T=0) == 0
    assert call(T=-1) == 1
    assert call(T=9) == 1                      # only decode windows
    assert call(x=0x4008) == 2
    assert call(wsb=16) == 3
    assert call(out=0x4000 + 256) == 1
    # the staging rows are part of the workspace: one sized for T holds every T' <= T
    assert B.moe_workspace_bytes(d, 8) >= B.moe_workspace_bytes(d, 3) > 0


@pytest.mark.parametrize("dims", [(2048, 512, 512, 10), (256, 128, 16, 2), (512, 512, 16, 2), (4096, 4096, 4096, 32),
                                  (256, 1024, 4096, 8)])
def test_workspace_size_never_shrinks_with_tokens(lib, dims):
    """A workspace sized for max_T must hold every call with T <= max_T (the router's K-split count and the
    prefill item size change with T, so this is not automatic)."""
    d = B.moe_dims(*dims)
    prev = 0
    for T in list(range(1, 300)) + [511, 512, 513, 1023, 1024, 1025, 2048, 3277, 4096, 8192, 32768]:
        need = lib.moe_workspace_bytes(ctypes.byref(d), T)
        assert need >= prev, (dims, T, need, prev)
        prev = need


@pytest.mark.parametrize("dims", [(128, 128, 1, 1), (4096, 4096, 16, 2), (256, 128, 65535, 32), (2048, 512, 512, 10),
                                  (384, 640, 5000, 4)])
def test_limits_accepted(lib, dims):
    """The edges of the stated limits: multiples of 128 up to 4096, up to 65535 experts, up to 32 per token."""
    d = B.moe_dims(*dims)
    H, I = dims[0], dims[1]
    assert B.moe_canonical_expert_bytes(d) == 3 * H * I // 32 * 10
    assert B.moe_packed_expert_bytes(d) >= B.moe_canonical_expert_bytes(d)
    assert B.moe_workspace_bytes(d, 8) > 0
