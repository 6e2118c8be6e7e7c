"""Seeded synthetic attention inputs shaped like Wan-class video-DiT attention.

This module only draws Q, K, V. It holds none of the method's arithmetic
(no permutation, pooling, scoring, selection or attention), so both the CUDA
path and the fp64 oracle can consume its tensors without sharing code.

Workloads (the latent grids of the pages' settings):
  * tiny           B1 H2 d64 fp32, grid 4x8x8, tiles 1x8x8, 64-token blocks,
                   Q,K,V ~ N(0,1), head 1's Q scaled by 3 (peakier logits),
                   p=0.9, k_min=1.
  * wan1.3b-480p   B1 H12 d128 bf16, grid 21x30x52 (480x832 video, 81 frames),
                   2x8x8 tiles, 128-token blocks, p=0.9, k_min=4,
                   per-head temperature ~ U[0.5, 4].
  * wan14b-480p    as above with H40 and temperature log-uniform in [0.3, 6].
  * wan14b-720p    B1 H40 d128 bf16, grid 21x45x80 (720p, 81 frames -> 21
                   latent frames x 3,600 tokens), 2x8x8 tiles, 128-token
                   blocks, p=0.95, k_min=8, temperature log-uniform [0.3, 6].
For the video workloads Q and K are N(0,1) noise plus 0.5 x a smooth 3-D
sin/cos positional code PE(t, y, x) shared by Q and K, so that nearby tokens
have similar queries and keys; Q of head h is multiplied by its temperature.
V ~ N(0,1). The code is a set of d random Fourier features over the
normalised grid coordinates u = (t/T, y/Hh, x/W):
    PE_c(u) = sqrt(2) * cos(2*pi * f_c . u + phi_c),
with f_c ~ N(0, F0^2 I_3) cycles per axis extent and phi_c ~ U[0, 2*pi), drawn
once from a fixed seed. Each channel has unit RMS, and PE(u) . PE(u') falls
off smoothly with the 3-D distance |u - u'|. F0 = 0.5 was chosen once, so
that the temperature range spreads per-head block density as widely as this
recipe allows (about 4% to 90% at p = 0.9), and is frozen.
"""

from __future__ import annotations

import dataclasses
import math

import torch

F0 = 0.5      # std of the code's frequencies, in cycles per axis extent
PE_SEED = 7   # fixed seed of the code's frequencies and phases


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    dtype: str                 # "bf16" or "fp32"
    grid: tuple                # (T, Hh, W)
    tile: tuple                # (tt, th, tw)
    block: int
    p: float
    k_min: int
    seed: int
    gen: str = "video"         # "video" (noise + PE, temperatures) or "gauss"
    temp: tuple = ("uniform", 1.0, 1.0)
    peaky_head: int = -1
    peaky_scale: float = 1.0

    @property
    def N(self) -> int:
        T, Hh, W = self.grid
        return T * Hh * W

    @property
    def nb(self) -> int:
        return -(-self.N // self.block)

    @property
    def grid6(self) -> tuple:
        return tuple(self.grid) + tuple(self.tile)

    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, "fp32", (4, 8, 8), (1, 8, 8), 64, 0.9, 1, seed=0,
                     gen="gauss", peaky_head=1, peaky_scale=3.0),
    "wan1.3b-480p": Workload("wan1.3b-480p", 1, 12, 128, "bf16", (21, 30, 52), (2, 8, 8), 128,
                             0.9, 4, seed=1, temp=("uniform", 0.5, 4.0)),
    "wan14b-480p": Workload("wan14b-480p", 1, 40, 128, "bf16", (21, 30, 52), (2, 8, 8), 128,
                            0.9, 4, seed=2, temp=("loguniform", 0.3, 6.0)),
    "wan14b-720p": Workload("wan14b-720p", 1, 40, 128, "bf16", (21, 45, 80), (2, 8, 8), 128,
                            0.95, 8, seed=3, temp=("loguniform", 0.3, 6.0)),
}


def sweep_workloads():
    """The 720p sweep: p x k_min x block size (64-token blocks use 1x8x8 tiles)."""
    base = WORKLOADS["wan14b-720p"]
    out = []
    for bs, tile in ((128, (2, 8, 8)), (64, (1, 8, 8))):
        for p in (0.5, 0.7, 0.9, 0.95, 0.99, 1.0):
            for k_min in (1, 4, 16):
                out.append(base.replace(name=f"wan14b-720p-bs{bs}-p{p}-k{k_min}",
                                        block=bs, tile=tile, p=p, k_min=k_min))
    return out


def temperatures(w: Workload) -> torch.Tensor:
    """Per-head Q temperatures, drawn on the CPU so they do not depend on the device."""
    g = torch.Generator(device="cpu").manual_seed(10_000 + w.seed)
    kind, lo, hi = w.temp
    u = torch.rand(w.H, generator=g, dtype=torch.float64)
    if kind == "uniform":
        t = lo + (hi - lo) * u
    elif kind == "loguniform":
        t = torch.exp(math.log(lo) + (math.log(hi) - math.log(lo)) * u)
    else:
        raise ValueError(kind)
    return t.to(torch.float32)


def positional_code(grid, d: int, device="cpu") -> torch.Tensor:
    """Smooth 3-D random-Fourier-feature code [T*Hh*W, d] (float32), unit RMS per channel."""
    T, Hh, W = grid
    g = torch.Generator(device="cpu").manual_seed(PE_SEED)
    freq = torch.randn(d, 3, generator=g, dtype=torch.float64) * F0
    phase = torch.rand(d, generator=g, dtype=torch.float64) * (2.0 * math.pi)
    axes = [torch.arange(n, dtype=torch.float64) / n for n in (T, Hh, W)]
    tg, yg, xg = torch.meshgrid(*axes, indexing="ij")
    u = torch.stack([tg.reshape(-1), yg.reshape(-1), xg.reshape(-1)], dim=-1)
    pe = math.sqrt(2.0) * torch.cos(2.0 * math.pi * (u @ freq.T) + phase)
    return pe.to(device=device, dtype=torch.float32)


def make_qkv(w: Workload, device="cpu"):
    """Draw (q, k, v) of shape [B, H, N, d] in the workload's dtype on ``device``.

    The draw is deterministic for a given (workload seed, device type). The
    oracle always receives the exact bytes the GPU path received (copied back
    to the host), so CPU and GPU generators need not agree.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.d)
    out_dt = w.torch_dtype()
    if w.gen == "gauss":
        q = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        k = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        v = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        if 0 <= w.peaky_head < w.H:
            q[:, w.peaky_head] *= w.peaky_scale
        return q.to(out_dt), k.to(out_dt), v.to(out_dt)
    pe = 0.5 * positional_code(w.grid, w.d, dev)
    tau = temperatures(w).to(dev).view(1, w.H, 1, 1)
    q = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
    q.add_(pe).mul_(tau)
    q = q.to(out_dt)
    k = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
    k = k.add_(pe).to(out_dt)
    v = torch.randn(shape, generator=g, device=dev, dtype=out_dt)
    return q, k, v
