"""Seeded synthetic inputs for the routed MoE layer over Q2 block-quantized experts.

This module only *draws* inputs: random activations, router weights, router
bias and random 2-bit codes with fp16 block scales, encoded in the canonical
Q2 block format.  It holds none of the layer's arithmetic (no dequantisation,
no routing, no FFN); the CPU oracle and the CUDA library each decode the same
bytes with their own code.

Workload shapes follow the pages' model: 48 layers x 512 routed experts, each
token routed to 10 experts plus 1 shared expert (Strata tuning page, section 2
"Strata 是什么", model table), prompts processed in 1024-token chunks (devlabs
page, section 1) or 32768-token chunks (`--prefill auto:32768`, Strata tuning
page, section 4), and a 1-3 token guess-and-check verify window (devlabs page,
section 1).  The hidden/intermediate sizes (2048 / 512) and the value
distributions are synthetic stand-ins: the pages ship no weights.

Canonical Q2 block (10 bytes): little-endian fp16 scale d, then 8 bytes qs;
element j (0..31) of the block is ``(qs[j >> 2] >> (2 * (j & 3))) & 3``.  An
expert is three matrices stored back to back, each row-major with blocks of
32 running along the contraction dimension:
  gate [I rows x H/32 blocks], up [I x H/32], down [H rows x I/32 blocks].
"""
from __future__ import annotations

import dataclasses
import numpy as np

QBLOCK = 32          # weights per block
QBLOCK_BYTES = 10    # fp16 scale + 8 bytes of 2-bit codes

# Router-bias strength for the Zipf(s=1.1)-skewed configurations.  Chosen so
# that, at T=1024 with seed 0, the hottest expert receives about 100 of the
# 10240 routed slots while every expert is still hit (checked by
# tests/test_inputs.py against the oracle's routing).
ZIPF_S = 1.1
ZIPF_BETA = 0.125
# A second, colder point: a heavier tail with many experts receiving 0-2 tokens.
ZIPF_BETA_COLD = 0.35


@dataclasses.dataclass(frozen=True)
class MoeConfig:
    name: str
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    tokens: int
    bias: str = "zero"          # "zero" | "zipf" | "zipf_cold"
    layers: int = 1
    rmsnorm: bool = False

    @property
    def expert_bytes(self) -> int:
        return canonical_expert_bytes(self.hidden, self.inter)


CONFIGS = {
    "tiny": MoeConfig("tiny layer H256 I128 E16 top2+1 T8", 256, 128, 16, 2, 8),
    "decode": MoeConfig("decode layer H2048 I512 E512 top10+1 T3", 2048, 512, 512, 10, 3),
    "prefill": MoeConfig("prefill layer H2048 I512 E512 top10+1 T1024 zipf", 2048, 512, 512, 10, 1024, "zipf"),
    "stack": MoeConfig("48-layer stack H2048 I512 E512 top10+1 T1024 zipf rmsnorm", 2048, 512, 512, 10, 1024,
                       "zipf", layers=48, rmsnorm=True),
    "prefill_32k": MoeConfig("4-layer prefill H2048 I512 E512 top10+1 T32768 zipf", 2048, 512, 512, 10, 32768,
                             "zipf", layers=4),
}


def canonical_expert_bytes(hidden: int, inter: int) -> int:
    nblk = (2 * inter * hidden + hidden * inter) // QBLOCK
    return nblk * QBLOCK_BYTES


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_x(cfg_or_tokens, hidden: int | None = None, seed: int = 0, slot: int = 0) -> np.ndarray:
    """Activations x ~ N(0,1) rounded to bf16; returns uint16 bits [T, H]."""
    if isinstance(cfg_or_tokens, MoeConfig):
        T, H = cfg_or_tokens.tokens, cfg_or_tokens.hidden
    else:
        T, H = int(cfg_or_tokens), int(hidden)
    rng = np.random.default_rng([seed, 1, slot])
    return f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))


def make_router(cfg: MoeConfig, seed: int = 0, layer: int = 0, bias: str | None = None):
    """Router weight Wr [E, H] fp32 ~ N(0, 0.02) and bias [E] fp32."""
    E, H = cfg.n_experts, cfg.hidden
    rng = np.random.default_rng([seed, 2, layer])
    w = (rng.standard_normal((E, H), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    kind = cfg.bias if bias is None else bias
    if kind == "zero":
        b = np.zeros(E, dtype=np.float32)
    else:
        beta = ZIPF_BETA if kind == "zipf" else ZIPF_BETA_COLD
        ranks = rng.permutation(E).astype(np.float64) + 1.0
        b = (beta * (-ZIPF_S * np.log(ranks))).astype(np.float32)
    return w, b


def make_expert(hidden: int, inter: int, seed: int, layer: int, expert: int) -> np.ndarray:
    """One expert's canonical Q2 bytes [expert_bytes] uint8.

    Codes are uniform in {0,1,2,3} (uniform random bytes give independent
    uniform 2-bit fields); scales are fp16(|N(0, 0.02)|).
    """
    nblk = (3 * inter * hidden) // QBLOCK
    rng = np.random.default_rng([seed, 3, layer, expert])
    d = np.abs(rng.standard_normal(nblk, dtype=np.float32) * np.float32(0.02)).astype(np.float16)
    qs = np.frombuffer(rng.bytes(nblk * 8), dtype=np.uint8).reshape(nblk, 8)
    out = np.empty((nblk, QBLOCK_BYTES), dtype=np.uint8)
    out[:, 0:2] = d.view(np.uint8).reshape(nblk, 2)
    out[:, 2:10] = qs
    return out.reshape(-1)


def make_experts(cfg: MoeConfig, seed: int = 0, layer: int = 0, experts=None) -> np.ndarray:
    """Canonical bytes for routed experts (default all E) stacked [n, expert_bytes]."""
    ids = range(cfg.n_experts) if experts is None else experts
    return np.stack([make_expert(cfg.hidden, cfg.inter, seed, layer, int(e)) for e in ids])


def make_shared(cfg: MoeConfig, seed: int = 0, layer: int = 0) -> np.ndarray:
    """The shared expert's canonical bytes [expert_bytes]; drawn as expert id E."""
    return make_expert(cfg.hidden, cfg.inter, seed, layer, cfg.n_experts)


def make_layer(cfg: MoeConfig, seed: int = 0, layer: int = 0, bias: str | None = None):
    """Everything one layer needs: dict of numpy arrays (x is drawn separately)."""
    w, b = make_router(cfg, seed, layer, bias)
    return {
        "router_w": w,
        "router_b": b,
        "experts": make_experts(cfg, seed, layer),
        "shared": make_shared(cfg, seed, layer),
    }


def make_layer_device(cfg: MoeConfig, seed: int = 0, layer: int = 0, device="cuda", bias: str | None = None):
    """A layer with the same distributions as make_layer, drawn on the GPU with torch's generator (fast enough
    for the benchmark's 48-layer stack; the parity tests use make_layer, whose values the oracle regenerates).
    Returns a dict of device tensors: router_w [E, H] fp32 ~ N(0, 0.02), router_b [E] fp32 (zero or the
    Zipf(s) bias over a seeded rank permutation), experts [E, expert_bytes] uint8 and shared [expert_bytes]
    uint8 in the canonical Q2 format (codes uniform in {0..3}, scales fp16(|N(0, 0.02)|))."""
    import torch

    E, H = cfg.n_experts, cfg.hidden
    g = torch.Generator(device=device)
    g.manual_seed(((seed * 1000003) ^ (layer * 7919) ^ 0x5EED) & 0x7FFFFFFFFFFF)
    w = torch.randn((E, H), generator=g, device=device, dtype=torch.float32) * 0.02
    kind = cfg.bias if bias is None else bias
    if kind == "zero":
        b = torch.zeros(E, dtype=torch.float32, device=device)
    else:
        beta = ZIPF_BETA if kind == "zipf" else ZIPF_BETA_COLD
        ranks = torch.randperm(E, generator=g, device=device).to(torch.float64) + 1.0
        b = (beta * (-ZIPF_S * torch.log(ranks))).to(torch.float32)
    nblk = (3 * cfg.inter * H) // QBLOCK

    def expert_blocks(n):
        d = (torch.randn((n * nblk,), generator=g, device=device, dtype=torch.float32) * 0.02).abs().to(torch.float16)
        qs = torch.randint(0, 256, (n * nblk, 8), generator=g, device=device, dtype=torch.uint8)
        out = torch.empty((n * nblk, QBLOCK_BYTES), dtype=torch.uint8, device=device)
        out[:, 0:2] = d.view(torch.uint8).view(n * nblk, 2)
        out[:, 2:] = qs
        return out.view(n, nblk * QBLOCK_BYTES)

    experts = torch.cat([expert_blocks(min(64, E - e0)) for e0 in range(0, E, 64)])
    shared = expert_blocks(1).view(-1)
    return {"router_w": w, "router_b": b, "experts": experts, "shared": shared}
