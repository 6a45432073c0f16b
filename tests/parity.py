"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gen import MoeConfig, make_layer, make_x

# BASELINE tolerances: routing sets bit-exact except near-ties; layer output
# max|dy| / max|y_oracle| <= 1e-2 with bf16 activations and fp32 accumulation.
GAP_TIE = 1e-5
Y_TOL = 1e-2
W_TOL = 1e-5


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits).view(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_dev_bf16(x_bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(device)


def build_layer(cfg: MoeConfig, seed=0, layer=0, bias=None, device="cuda"):
    from bit_block_quantized_moe_b200 import Q2MoeLayer

    w = make_layer(cfg, seed=seed, layer=layer, bias=bias)
    L = Q2MoeLayer(cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k, w["router_w"], w["router_b"], w["experts"],
                   w["shared"], device=device)
    return L, w


def gpu_forward(L, x_bits: np.ndarray):
    T = x_bits.shape[0]
    k = L.dims.top_k
    xd = to_dev_bf16(x_bits, L.device)
    idx = torch.full((T, k), -1, dtype=torch.int32, device=L.device)
    wts = torch.zeros((T, k), dtype=torch.float32, device=L.device)
    out = L.forward(xd, topk_idx=idx, topk_w=wts)
    torch.cuda.synchronize()
    L.check_status()
    return bf16_to_f64(out.cpu().numpy()), idx.cpu().numpy(), wts.cpu().numpy()


def check_routing(idx_gpu, w_gpu, idx_orc, w_orc, gap_orc):
    """Index sets bit-exact except tokens whose k-th/(k+1)-th gap < GAP_TIE; returns the flagged tokens."""
    flagged = []
    for t in range(idx_gpu.shape[0]):
        if set(idx_gpu[t].tolist()) != set(idx_orc[t].tolist()):
            assert gap_orc[t] < GAP_TIE, f"token {t}: routing differs with gap {gap_orc[t]:.3e}"
            flagged.append(t)
        else:
            og, oo = np.argsort(idx_gpu[t]), np.argsort(idx_orc[t])
            assert np.max(np.abs(w_gpu[t][og] - w_orc[t][oo])) <= W_TOL, f"token {t}: weights differ"
    assert np.all(np.abs(w_gpu.sum(axis=1) - 1.0) < 1e-5)
    return flagged


def check_layer(cfg: MoeConfig, w, x_bits, y_gpu, idx_gpu, w_gpu, tokens=None):
    """Compare the GPU layer with the oracle on `tokens` (default all).  Tokens
    with a different routing set must be near-ties; for them the oracle is
    re-run with the GPU's set.  Returns (max-rel error, rel L2, flagged)."""
    if tokens is None:
        tokens = np.arange(x_bits.shape[0])
    xs = x_bits[tokens]
    y_orc, idx_orc, w_orc, gap = oracle.layer(xs, w["router_w"], w["router_b"], w["experts"], w["shared"], cfg.top_k,
                                              cfg.inter)
    flagged = check_routing(idx_gpu[tokens], w_gpu[tokens], idx_orc, w_orc, gap)
    if flagged:
        f = np.array(flagged)
        y_f, _, _, _ = oracle.layer(xs[f], w["router_w"], w["router_b"], w["experts"], w["shared"], cfg.top_k,
                                    cfg.inter, forced_idx=idx_gpu[tokens][f])
        y_orc[f] = y_f
    yg = y_gpu[tokens]
    denom = np.max(np.abs(y_orc))
    err = np.max(np.abs(yg - y_orc)) / denom if denom > 0 else np.max(np.abs(yg))
    rel_l2 = np.linalg.norm(yg - y_orc) / max(np.linalg.norm(y_orc), 1e-300)
    assert err <= Y_TOL, f"max|dy|/max|y| = {err:.3e} > {Y_TOL}"
    return err, rel_l2, flagged
