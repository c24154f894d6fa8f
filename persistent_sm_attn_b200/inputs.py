"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws random numbers and names workloads; it holds none of
the attention arithmetic, so the CUDA path and the CPU oracle can both consume
its tensors without sharing any computation.

Recipe.  Workload ``i`` (0-based) uses seed ``1000 + i + 1`` for a
``torch.Generator`` on the requested device.  Q, K, V and dO are drawn in that
order as float32 standard normals of shape [B, H, S, D], multiplied by sigma and
rounded to bf16 (round to nearest even).  The softmax scale is 1/sqrt(D).  O and
LSE come from the library's forward on the same inputs.  The pages name no
dataset; these shapes stand in for the LLM and diffusion-transformer attention
layers the pages evaluate (DASH summary §4).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    causal: bool
    sigma: float
    schedules: tuple  # schedules compared on this workload, the best measured first

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def n_tiles(self) -> int:
        return self.S // 128

    @property
    def flops(self) -> float:
        """Backward FLOPs: 5 matrix products of 2*S*S*D each per head (half
        of that with a causal mask)."""
        f = 10.0 * self.B * self.H * self.S * self.S * self.D
        return f / 2 if self.causal else f


WORKLOADS = (
    Workload("full_b1_h2_s256_d64", 1, 2, 256, 64, False, 1.0, ("shift",)),
    Workload("full_b2_h16_s4096_d128", 2, 16, 4096, 128, False, 1.0,
             ("shift", "descending", "naive_asc", "atomic")),
    Workload("causal_b2_h32_s8192_d128", 2, 32, 8192, 128, True, 1.0,
             ("sym_shift", "descending", "naive_asc", "atomic")),
    Workload("causal_b4_h32_s16384_d64", 4, 32, 16384, 64, True, 1.0,
             ("sym_shift", "descending", "atomic")),
    Workload("full_b1_h24_s16384_d128", 1, 24, 16384, 128, False, 0.5,
             ("descending", "shift", "atomic")),
)


def seed_of(index: int) -> int:
    return 1000 + index + 1


def draw(B, H, S, D, sigma=1.0, seed=0, device="cpu"):
    """Q, K, V, dO as bf16 [B,H,S,D] tensors on ``device``."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = []
    for _ in range(4):
        x = torch.randn((B, H, S, D), generator=g, device=device, dtype=torch.float32)
        out.append((x * sigma).to(torch.bfloat16))
    return tuple(out)


def workload_inputs(index: int, device="cpu"):
    w = WORKLOADS[index]
    return draw(w.B, w.H, w.S, w.D, w.sigma, seed_of(index), device)


def sample_heads(B: int, H: int, n: int, seed: int):
    """n distinct (b, h) heads chosen by a seeded generator (for sampled parity
    at sizes the oracle cannot finish in full)."""
    g = torch.Generator()
    g.manual_seed(seed)
    idx = torch.randperm(B * H, generator=g)[: min(n, B * H)].tolist()
    return sorted((i // H, i % H) for i in idx)
