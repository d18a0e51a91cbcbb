"""Seeded synthetic inputs shaped like the latents of a Wan2.1/2.2-class video DiT.

This module holds no SageSLA arithmetic. It only draws Q, K and V, so that the CUDA
path and the CPU oracle read byte-identical bf16 tensors.

The pages (TurboDiffusion write-ups, "Performance Benchmarks" table of the English
write-up) quote Wan2.1-T2V-1.3B-480P and Wan-14B-720P runs; no latent tensors are
published, so seeded fields of the same shape stand in for them.

Recipe, per (batch, head), in this fixed draw order from one
``numpy.random.default_rng(seed)`` (PCG64) stream:

1. Four sinusoids. Each has integer frequencies (f_t, f_h, f_w) drawn uniformly from
   {0,1,2,3} (redrawn while all three are 0) and a phase drawn from U[0, 2*pi).
   Component c is F_c(t,h,w) = sin(2*pi*(f_t*t/T + f_h*h/Hg + f_w*w/W) + phase_c).
2. Three projections P_q, P_k, P_v of shape 4 x d, entries N(0, 1/4) (variance).
3. X = F @ P_x + N(0, 1/2) noise (variance), for X in Q, K, V, in that order.
4. K += bias, one N(0, 4) draw (variance) per channel.

Tokens are ordered row-major over (t, h, w). Values are produced in float64 and
rounded once to bf16 by torch (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    """One synthetic SageSLA workload: shape, token grid and sparsity ratios."""

    name: str
    B: int
    H: int
    grid: tuple  # (T, Hg, W) latent grid; N = T*Hg*W
    rho: float
    nu: float
    seeds: tuple = (0,)
    d: int = HEAD_DIM

    @property
    def N(self) -> int:
        t, h, w = self.grid
        return t * h * w


# Workloads for parity and measurement. Shapes follow the Wan latent grids (480p:
# 21x30x52 tokens, 720p: 21x45x80) with head dim 128: the 1.3B model has 12 heads, the
# 14B models 40. Second workloads on the same kernels: "480p_14b" (Wan2.1-14B at 480p),
# "480p_topk015" (--sla_topk 0.15 on the 1.3B layer) and "720p_i2v" (Wan2.2-I2V-A14B at
# 720p: its DiT sees the same 21x45x80 token grid and 40 heads as the 14B T2V layer, the
# image condition entering through the input channels, so only the seed differs).
SWEEP_RHOS = (1.0, 0.5, 0.2, 0.1, 0.05)


def sweep_workload(rho: float) -> Workload:
    """480p-shaped sweep point: B=2, nu=(1-rho)/2, seeds 0 and 1."""
    return Workload(f"sweep_rho{rho:g}", 2, 12, (21, 30, 52), rho, (1.0 - rho) / 2.0, (0, 1))


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, (4, 16, 16), 0.25, 0.25),
    "dense": Workload("dense", 1, 12, (4, 32, 32), 1.0, 0.0),
    "480p": Workload("480p", 1, 12, (21, 30, 52), 0.10, 0.45),
    "720p": Workload("720p", 1, 40, (21, 45, 80), 0.10, 0.45),
    "480p_14b": Workload("480p_14b", 1, 40, (21, 30, 52), 0.10, 0.45),
    "480p_topk015": Workload("480p_topk015", 1, 12, (21, 30, 52), 0.15, 0.45),
    "720p_i2v": Workload("720p_i2v", 1, 40, (21, 45, 80), 0.10, 0.45, (1,)),
}
WORKLOADS.update({f"sweep_rho{r:g}": sweep_workload(r) for r in SWEEP_RHOS})


def _head_fields(rng: np.random.Generator, grid, d: int):
    T, Hg, W = grid
    t = np.arange(T, dtype=np.float64)[:, None, None]
    h = np.arange(Hg, dtype=np.float64)[None, :, None]
    w = np.arange(W, dtype=np.float64)[None, None, :]
    comps = []
    for _ in range(4):
        while True:
            f = rng.integers(0, 4, size=3)
            if f.any():
                break
        phase = rng.uniform(0.0, 2.0 * math.pi)
        arg = 2.0 * math.pi * (f[0] * t / T + f[1] * h / Hg + f[2] * w / W) + phase
        comps.append(np.sin(arg).reshape(-1))
    F = np.stack(comps, axis=1)  # [N, 4]
    proj = [rng.normal(0.0, 0.5, size=(4, d)) for _ in range(3)]
    n = F.shape[0]
    out = []
    for P in proj:
        out.append(F @ P + rng.normal(0.0, math.sqrt(0.5), size=(n, d)))
    out[1] += rng.normal(0.0, 2.0, size=(d,))[None, :]
    return out


def make_qkv(B: int, H: int, grid, seed: int = 0, d: int = HEAD_DIM):
    """Draw bf16 Q, K, V of shape [B, H, N, d] (CPU tensors) from the recipe above."""
    rng = np.random.default_rng(seed)
    N = grid[0] * grid[1] * grid[2]
    q = torch.empty(B, H, N, d, dtype=torch.bfloat16)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    for b in range(B):
        for hh in range(H):
            xq, xk, xv = _head_fields(rng, grid, d)
            q[b, hh] = torch.from_numpy(xq).to(torch.bfloat16)
            k[b, hh] = torch.from_numpy(xk).to(torch.bfloat16)
            v[b, hh] = torch.from_numpy(xv).to(torch.bfloat16)
    return q, k, v


def make_workload_qkv(wl: Workload, seed: int | None = None):
    return make_qkv(wl.B, wl.H, wl.grid, wl.seeds[0] if seed is None else seed, wl.d)


def make_random_qkv(B: int, H: int, N: int, seed: int = 0, d: int = HEAD_DIM,
                    k_bias: float = 2.0, scale: float = 1.0):
    """Plain N(0, scale^2) Q/K/V with an N(0, k_bias^2) per-channel K offset (edge cases)."""
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) * scale)
    k = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) * scale)
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float64)
    k = k + torch.randn(B, H, 1, d, generator=g, dtype=torch.float64) * k_bias
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
