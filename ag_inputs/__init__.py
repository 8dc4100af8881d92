"""Seeded synthetic inputs for the pair-bias multi-query attention workloads.

This module is shared by the tests, the benchmark, the oracle checks and the
GPU path.  It holds none of the method's arithmetic: it only draws random
numbers with torch's CPU generator and describes workload sizes.

Workload shapes follow the page "Making Full-Context AlphaGenome Fit on an
RTX 3090" (section "Profiling pointed at one very large object": 8,192
transformer positions at full context, eight query heads sharing one K/V
head; section "Why stock FlashAttention was not a drop-in replacement":
D = 128, compact bias with one cell per 16 positions, cap 5) and the page
"From Code to Cure: How AlphaGenome Decodes the 'Dark Matter' of DNA"
(section "The Architecture": 128 bp per sequence position and 2,048 bp per
pair cell, so a 1,048,576 bp input gives L = 8192 and P = 512).

Draw order per seed: q, k, v (float32 N(0,1), then rounded to bf16 with
round-to-nearest-even), then either the compact bias [H,P,P] or the pair
representation [P,P,Cp] followed by W [Cp,H].  No public dataset is involved;
the pages measured on none for the attention itself.
"""
from __future__ import annotations

import math
import random
from dataclasses import dataclass, field

import torch

H_DEFAULT = 8
D_DEFAULT = 128
BLOCK_DEFAULT = 16
CP_DEFAULT = 128


@dataclass(frozen=True)
class Workload:
    """One attention workload (one layer)."""
    name: str
    B: int
    L: int
    seed: int
    cap: float = 5.0
    H: int = H_DEFAULT
    D: int = D_DEFAULT
    Dv: int = D_DEFAULT
    block: int = BLOCK_DEFAULT
    bias_mode: str = "direct"      # "direct": bias drawn; "pair": projected
    bias_std: float = 1.0
    Cp: int = CP_DEFAULT
    w_std: float = 1.0 / math.sqrt(CP_DEFAULT)

    @property
    def P(self) -> int:
        return self.L // self.block

    def attn_flops(self) -> float:
        """Tensor FLOPs counted for one call: 2*B*H*L^2*(D + Dv) = 4BHL^2D."""
        return 2.0 * self.B * self.H * self.L * self.L * (self.D + self.Dv)

    def attn_bytes(self) -> int:
        """Algorithmic HBM bytes of one attention call: each input read once
        (q, k, v bf16; compact bias fp32) and each output written once
        (out, lse fp32)."""
        B, H, L, D, Dv, P = self.B, self.H, self.L, self.D, self.Dv, self.P
        return (2 * B * H * L * D + 2 * B * L * D + 2 * B * L * Dv
                + 4 * H * P * P + 4 * B * H * L * Dv + 4 * B * H * L)

    def project_bytes(self) -> int:
        """Algorithmic HBM bytes of one projection: pair + W read, bias written."""
        P, Cp, H = self.P, self.Cp, self.H
        return 4 * P * P * Cp + 4 * Cp * H + 4 * H * P * P


@dataclass(frozen=True)
class Stack:
    """Several independent layers run back to back."""
    name: str
    layers: tuple = field(default_factory=tuple)


def _layer_cap(seed: int) -> float:
    return random.Random(seed).choice([5.0, 10.0, 30.0])


def nine_block_stack() -> Stack:
    """Nine independent L=8192, B=2 layers, seeds 10..18, pair-projected bias,
    cap drawn per layer from {5, 10, 30} with random.Random(seed)."""
    layers = tuple(
        Workload(name=f"nine_block_layer{l}", B=2, L=8192, seed=10 + l,
                 cap=_layer_cap(10 + l), bias_mode="pair")
        for l in range(9))
    return Stack(name="nine_block", layers=layers)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, L=512, seed=0, bias_std=1.0),
    "short": Workload("short", B=1, L=2048, seed=1, bias_std=1.0),
    "mid": Workload("mid", B=1, L=4096, seed=2, bias_std=0.5),
    "full": Workload("full", B=1, L=8192, seed=3, bias_mode="pair"),
}


def make_inputs(w: Workload) -> dict:
    """Draw one layer's inputs on the CPU.

    Returns a dict with q [B,H,L,D] bf16, k [B,L,D] bf16, v [B,L,Dv] bf16 and
    either bias [H,P,P] fp32 (direct mode) or pair [P,P,Cp] fp32 and
    W [Cp,H] fp32 (pair mode).
    """
    g = torch.Generator(device="cpu").manual_seed(int(w.seed))
    q = torch.randn(w.B, w.H, w.L, w.D, generator=g).to(torch.bfloat16)
    k = torch.randn(w.B, w.L, w.D, generator=g).to(torch.bfloat16)
    v = torch.randn(w.B, w.L, w.Dv, generator=g).to(torch.bfloat16)
    out = {"q": q, "k": k, "v": v}
    if w.bias_mode == "direct":
        out["bias"] = torch.randn(w.H, w.P, w.P, generator=g) * w.bias_std
    elif w.bias_mode == "pair":
        out["pair"] = torch.randn(w.P, w.P, w.Cp, generator=g)
        out["W"] = torch.randn(w.Cp, w.H, generator=g) * w.w_std
    else:
        raise ValueError(w.bias_mode)
    return out


def random_case(B: int, H: int, L: int, D: int, Dv: int, block: int,
                seed: int, bias_std: float = 1.0, qk_std: float = 1.0,
                dtype=torch.bfloat16, batched_bias: bool = False) -> dict:
    """Small seeded case with free sizes (tests).  Same draw order as
    make_inputs: q, k, v, then bias.  L need not be a multiple of the block
    (P = ceil(L / block) compact cells per side); batched_bias draws one bias
    per batch item, [B, H, P, P], instead of one shared [H, P, P]."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    P = -(-L // block)
    q = (torch.randn(B, H, L, D, generator=g) * qk_std).to(dtype)
    k = (torch.randn(B, L, D, generator=g) * qk_std).to(dtype)
    v = torch.randn(B, L, Dv, generator=g).to(dtype)
    shape = (B, H, P, P) if batched_bias else (H, P, P)
    bias = torch.randn(*shape, generator=g) * bias_std
    return {"q": q, "k": k, "v": v, "bias": bias}


def sample_rows(B: int, H: int, L: int, n: int, seed: int) -> torch.Tensor:
    """n distinct (b, h, i) triples, always including the first and last
    query of the first and last batch, drawn with a seeded generator."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    total = B * H * L
    n = min(n, total)
    flat = torch.randperm(total, generator=g)[:n]
    fixed = torch.tensor([0, L - 1, total - L, total - 1], dtype=torch.long)
    flat = torch.unique(torch.cat([fixed.clamp(0, total - 1), flat]))
    b = flat // (H * L)
    h = (flat // L) % H
    i = flat % L
    return torch.stack([b, h, i], dim=1)
