"""Q2MoeLayer: owns the device buffers of one layer and calls the C ABI."""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B


class Q2MoeLayer:
    """One routed MoE layer: router (fp32), packed routed experts and packed shared expert.

    Buffers live on ``device``; ``forward`` calls ``moe_layer_forward`` once.
    The canonical Q2 bytes are copied to the device, repacked there by
    ``moe_pack_q2`` and released.
    """

    def __init__(self, hidden: int, inter: int, n_experts: int, top_k: int, router_w, router_b, experts_canon,
                 shared_canon, device="cuda", max_tokens: int = 0):
        self.dims = B.moe_dims(hidden, inter, n_experts, top_k)
        self.device = torch.device(device)
        self.router_w = self._f32(router_w)
        self.router_b = None if router_b is None else self._f32(router_b)
        pe = B.moe_packed_expert_bytes(self.dims)
        ce = B.moe_canonical_expert_bytes(self.dims)
        if pe == 0 or ce == 0:
            raise ValueError("unsupported layer dimensions")
        self.experts = torch.empty(n_experts * pe, dtype=torch.uint8, device=self.device)
        self.shared = torch.empty(pe, dtype=torch.uint8, device=self.device)
        self._pack(experts_canon, n_experts, ce, self.experts)
        self._pack(shared_canon, 1, ce, self.shared)
        self.workspace = None
        self._ws_T = -1
        if max_tokens:
            self.reserve(max_tokens)

    def _f32(self, a):
        if isinstance(a, torch.Tensor):
            return a.detach().to(self.device, torch.float32).contiguous()
        return torch.as_tensor(np.ascontiguousarray(a, dtype=np.float32)).to(self.device)

    def _pack(self, canon, n, ce, dst):
        if isinstance(canon, torch.Tensor):
            src = canon.detach().reshape(-1)
            assert src.dtype == torch.uint8
        else:
            src = torch.as_tensor(np.ascontiguousarray(canon, dtype=np.uint8).reshape(-1))
        assert src.numel() == n * ce
        # pack in slices to bound the temporary device copy
        per = max(1, (256 << 20) // ce)
        pe = B.moe_packed_expert_bytes(self.dims)
        for s in range(0, n, per):
            m = min(per, n - s)
            tmp = src[s * ce:(s + m) * ce].to(self.device)
            B.moe_pack_q2(self.dims, tmp, m, dst[s * pe:(s + m) * pe])
        torch.cuda.synchronize(self.device)

    def reserve(self, T: int):
        if T > self._ws_T:
            nbytes = B.moe_workspace_bytes(self.dims, T)
            self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
            self._ws_T = T

    def forward(self, x, out=None, topk_idx=None, topk_w=None, stream=None):
        """x: [T, hidden] bf16 (torch.bfloat16 or int16 bit patterns) on device."""
        T = x.shape[0]
        self.reserve(T)
        if out is None:
            out = torch.empty_like(x)
        B.moe_layer_forward(self.dims, x, self.router_w, self.router_b, self.experts, self.shared, out, T,
                            self.workspace, topk_idx, topk_w, stream)
        return out

    def forward_host(self, x_host, out_host=None, topk_idx=None, topk_w=None, stream=None):
        """x_host: [T <= 8, hidden] bf16 bit patterns in page-locked host memory; the output goes to out_host
        (page-locked, allocated if None), complete once the stream has passed the call."""
        T = x_host.shape[0]
        self.reserve(T)
        if out_host is None:
            out_host = torch.empty(x_host.shape, dtype=x_host.dtype).pin_memory()
        B.moe_layer_forward_host(self.dims, x_host, self.router_w, self.router_b, self.experts, self.shared, out_host,
                                 T, self.workspace, topk_idx, topk_w, stream)
        return out_host

    def forward_residual(self, x_norm, resid, x_norm_out, eps=1e-6, topk_idx=None, topk_w=None, stream=None):
        """One stacked layer: resid += layer(x_norm); x_norm_out = bf16(RMSNorm(resid))."""
        T = x_norm.shape[0]
        self.reserve(T)
        B.moe_layer_forward_residual(self.dims, x_norm, self.router_w, self.router_b, self.experts, self.shared, resid,
                                     x_norm_out, T, self.workspace, eps, topk_idx, topk_w, stream)
        return x_norm_out

    def experts_forward(self, x, topk_idx, topk_w, out=None, stream=None):
        T = x.shape[0]
        self.reserve(T)
        if out is None:
            out = torch.empty_like(x)
        B.moe_experts_forward(self.dims, x, topk_idx, topk_w, self.experts, self.shared, out, T, self.workspace,
                              stream)
        return out

    def route(self, x, topk_idx=None, topk_w=None, stream=None):
        T = x.shape[0]
        self.reserve(T)
        k = self.dims.top_k
        if topk_idx is None:
            topk_idx = torch.empty((T, k), dtype=torch.int32, device=self.device)
        if topk_w is None:
            topk_w = torch.empty((T, k), dtype=torch.float32, device=self.device)
        B.moe_route(self.dims, x, self.router_w, self.router_b, T, topk_idx, topk_w, self.workspace, stream)
        return topk_idx, topk_w

    def check_status(self, stream=None):
        B.moe_check_status(self.workspace, stream)
