"""Dispatch integers bit-exact: the CUDA dispatch (moe_dispatch, through the C ABI) against numpy on the
oracle's routing.  counts = bincount of the routed experts, offsets = their exclusive prefix sum, perm = numpy's
stable argsort of the flat slot list by expert (slots of one expert in ascending slot order), inv its inverse.
A dispatch that sends a slot to the right expert in the wrong order leaves the layer's sums unchanged (up to
rounding), so only this comparison sees it."""
import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, MoeConfig, make_router, make_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__

    __graft_entry__.build()
    assert torch.cuda.is_available()


def _dispatch(dims, idx_np, ws=None):
    import bit_block_quantized_moe_b200 as M

    T, k = idx_np.shape
    E = dims.n_experts
    if ws is None:
        ws = torch.zeros(M.moe_workspace_bytes(dims, T), dtype=torch.uint8, device="cuda")
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    M.moe_dispatch(dims, idx, T, counts, offsets, perm, inv, ws)
    torch.cuda.synchronize()
    return counts.cpu().numpy(), offsets.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy(), ws


def _expected(idx_np, E):
    flat = idx_np.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    perm = np.argsort(flat, kind="stable")
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return counts, offsets, perm, inv


@pytest.mark.parametrize("T", [13, 1024, 32768])
def test_dispatch_integers_bit_exact_on_oracle_routing(T):
    import bit_block_quantized_moe_b200 as M

    cfg = CONFIGS["prefill"]
    Wr, b = make_router(cfg, seed=0)
    x = make_x(T, cfg.hidden, seed=500 + T)
    idx_o, _, _, _ = oracle.route(x, Wr, b, cfg.top_k)
    dims = M.moe_dims(cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k)
    counts, offsets, perm, inv, ws = _dispatch(dims, idx_o)
    c, o, p, iv = _expected(idx_o, cfg.n_experts)
    assert np.array_equal(counts, c)
    assert np.array_equal(offsets, o)
    assert np.array_equal(perm, p)
    assert np.array_equal(inv, iv)
    M.moe_check_status(ws)


def test_dispatch_skewed_and_empty_experts():
    """Cold-tail routing (most experts empty, a few very hot) and a tiny layer whose experts are all hit."""
    import bit_block_quantized_moe_b200 as M

    rng = np.random.default_rng(1)
    for (H, I, E, k, T) in [(2048, 512, 512, 10, 777), (256, 128, 16, 2, 5), (256, 128, 16, 16, 40)]:
        p = np.arange(E, dtype=np.float64) + 1.0
        p = p ** -3.0
        p /= p.sum()
        idx = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
        dims = M.moe_dims(H, I, E, k)
        counts, offsets, perm, inv, ws = _dispatch(dims, idx)
        c, o, pp, iv = _expected(idx, E)
        assert np.array_equal(counts, c) and np.array_equal(offsets, o)
        assert np.array_equal(perm, pp) and np.array_equal(inv, iv)
        M.moe_check_status(ws)


def test_dispatch_bad_index_sets_status():
    import bit_block_quantized_moe_b200 as M
    from bit_block_quantized_moe_b200 import MoeError

    dims = M.moe_dims(256, 128, 16, 2)
    idx = np.array([[0, 1], [2, 99], [3, 4]], dtype=np.int32)
    counts, offsets, perm, inv, ws = _dispatch(dims, idx)
    with pytest.raises(MoeError) as e:
        M.moe_check_status(ws)
    assert e.value.code == 6
    assert inv[3] == -1 and offsets[-1] == 5  # the bad slot is left out
    good = np.array([0, 1, 2, 4, 5])
    c, o, pp, iv = _expected(idx.reshape(-1)[good].reshape(-1, 1), 16)
    assert np.array_equal(counts, c)
    assert np.array_equal(perm[:5], good[pp])
