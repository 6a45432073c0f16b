"""moe_route_noalloc: routing for callers that cannot allocate device memory
(engines whose device memory is reserved up front by their own pool, plug-ins
inside a framework that owns every allocation, or loops that cannot afford an
allocation's device synchronisation).  Its scratch is a static
device array inside the library; this checks it and moe_route, which uses a
caller-provided workspace, against the oracle on two calls in a row.  With more
than 8 tokens the two entry points use different router kernels (the workspace
one holds the split router weights for the tcgen05 router), so their routing is
only required to agree with the oracle's up to near-ties.  Collected last on
purpose."""
import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, make_router, make_x
from parity import check_routing

pytestmark = pytest.mark.gpu


def test_noalloc_route_matches_workspace_route():
    import __graft_entry__

    __graft_entry__.build()
    import bit_block_quantized_moe_b200 as M
    from bit_block_quantized_moe_b200 import binding as B

    cfg = CONFIGS["prefill"]
    dims = M.moe_dims(cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k)
    Wr, b = make_router(cfg, seed=0)
    Wd, bd = torch.from_numpy(Wr).cuda(), torch.from_numpy(b).cuda()
    ws = torch.zeros(M.moe_workspace_bytes(dims, 512), dtype=torch.uint8, device="cuda")
    for call, T in enumerate((3, 512)):  # two calls in a row, different sizes
        x = torch.from_numpy(make_x(T, cfg.hidden, seed=300 + call).view(np.int16)).cuda()
        idx_a = torch.full((T, cfg.top_k), -1, dtype=torch.int32, device="cuda")
        w_a = torch.zeros((T, cfg.top_k), dtype=torch.float32, device="cuda")
        idx_b, w_b = torch.full_like(idx_a, -2), torch.full_like(w_a, -1.0)
        M.moe_route(dims, x, Wd, bd, T, idx_a, w_a, ws)
        M.moe_route_noalloc(dims, x, Wd, bd, T, idx_b, w_b)
        torch.cuda.synchronize()
        x_np = x.cpu().numpy().view(np.uint16)
        idx_o, w_o, gap, _ = oracle.route(x_np, Wr, b, cfg.top_k)
        check_routing(idx_a.cpu().numpy(), w_a.cpu().numpy(), idx_o, w_o, gap)
        check_routing(idx_b.cpu().numpy(), w_b.cpu().numpy(), idx_o, w_o, gap)
        if T <= 8:  # same router kernel on both sides: identical results
            assert torch.equal(idx_a, idx_b) and torch.equal(w_a, w_b), f"call {call}: results differ"

    # sizes beyond the static scratch are rejected before any launch
    T_big = 262144 // cfg.n_experts + 1
    x = torch.zeros((T_big, cfg.hidden), dtype=torch.int16, device="cuda")
    idx = torch.zeros((T_big, cfg.top_k), dtype=torch.int32, device="cuda")
    w = torch.zeros((T_big, cfg.top_k), dtype=torch.float32, device="cuda")
    with pytest.raises(B.MoeError) as e:
        M.moe_route_noalloc(dims, x, Wd, bd, T_big, idx, w)
    assert e.value.code == 3  # MOE_ERR_WORKSPACE
