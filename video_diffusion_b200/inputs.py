"""Seeded synthetic attention inputs shaped like video-DiT attention calls.

This module only draws random numbers and filters them; it holds none of the
attention method's arithmetic.  It is the one piece shared by the CUDA path's
callers (tests, bench) and the oracle's callers.

Recipe (per batch entry and head):
  1. draw an iid N(0, 1) field G0 of shape [t, h, w, d] on the latent grid;
  2. blur it with a Gaussian of sigma = 2 cells, truncated at radius 8,
     separably along t, h and w, with half-sample-symmetric ("reflect")
     boundaries; axes of length 1 are left alone;
  3. divide every channel by its standard deviation over the grid -> G;
  4. Q = G + 0.5 N, K = G + 0.5 N', V ~ N(0, 1), tokens in raster t-h-w order;
  5. optionally append text-like tokens whose Q, K and V are iid N(0, 1).
Draw order per head: G0, N, N', V, then the text Q, K, V.  Inputs are made in
float32 and cast once to the requested dtype.

The pages measure on Wan 2.1-14B and HunyuanVideo-13B text-to-video at 720p
(81 and 129 frames); those weights and prompts are not available, so these
fields stand in for the query/key/value activations, at the same latent grids
(21 x 45 x 80 and 33 x 45 x 80).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

NEG_INF = -math.inf


@dataclass(frozen=True)
class Workload:
    """One attention-call shape with the betas it is exercised at."""

    name: str
    dtype: torch.dtype
    batch: int
    heads: int
    d: int
    grid: tuple  # (t, h, w) latent grid, raster order
    text_tokens: int
    block: int  # Bq = Bk
    betas: tuple
    seed: int
    notes: str = field(default="")

    @property
    def L(self) -> int:
        t, h, w = self.grid
        return t * h * w + self.text_tokens

    @property
    def n_blocks(self) -> int:
        return -(-self.L // self.block)

    def dense_flops(self) -> float:
        """4 b H L^2 d: QK^T plus PV of dense attention."""
        return 4.0 * self.batch * self.heads * float(self.L) ** 2 * self.d


WORKLOADS = {
    "tiny-fp32": Workload(
        "tiny-fp32 (1 head, L=1024 on 4x16x16, d=64, B=64)",
        torch.float32, 1, 1, 64, (4, 16, 16), 0, 64, (NEG_INF, 0.5, 1.04), 1000),
    "image-dit": Workload(
        "image-DiT (24 heads, L=16384 on 1x128x128, d=128, B=128)",
        torch.bfloat16, 1, 24, 128, (1, 128, 128), 0, 128, (0.5, 1.04, 1.5), 1001),
    "wan-480p": Workload(
        "Wan2.1-14B 480p (40 heads, L=32760 on 21x30x52, d=128, B=128)",
        torch.bfloat16, 1, 40, 128, (21, 30, 52), 0, 128, (1.04,), 1002),
    "wan-720p": Workload(
        "Wan2.1-14B 720p (40 heads, L=75600 on 21x45x80, d=128, B=128)",
        torch.bfloat16, 1, 40, 128, (21, 45, 80), 0, 128, (NEG_INF, 0.5, 1.04, 1.5, 2.0), 1003),
    "hunyuan-720p": Workload(
        "HunyuanVideo-13B 720p (24 heads, L=118800+256 text on 33x45x80, d=128, B=128)",
        torch.bfloat16, 1, 24, 128, (33, 45, 80), 256, 128, (1.04, 1.5), 1004),
    # image-DiT geometry with 64-wide heads (the head width of several image DiTs)
    "image-dit-d64": Workload(
        "image-DiT d=64 heads (24 heads, L=16384 on 1x128x128, d=64, B=128)",
        torch.bfloat16, 1, 24, 64, (1, 128, 128), 0, 128, (0.5, 1.04, 1.5), 1005),
}


def gaussian_filter_matrix(n: int, sigma: float = 2.0, radius: int = 8, dtype=torch.float64) -> torch.Tensor:
    """n x n matrix F with (F x)[i] = sum_k w_k x[reflect(i + k)], |k| <= radius.

    reflect() is half-sample symmetric: ... c b a | a b c ... | c b a ...,
    applied repeatedly, so any radius works for any n >= 1.
    """
    ks = torch.arange(-radius, radius + 1, dtype=torch.float64)
    w = torch.exp(-0.5 * (ks / sigma) ** 2)
    w = w / w.sum()
    F = torch.zeros(n, n, dtype=torch.float64)
    for i in range(n):
        for k, wk in zip(range(-radius, radius + 1), w.tolist()):
            p = (i + k) % (2 * n)
            if p >= n:
                p = 2 * n - 1 - p
            F[i, p] += wk
    return F.to(dtype)


def smooth_field(grid, d: int, gen: torch.Generator, device, sigma: float = 2.0, radius: int = 8) -> torch.Tensor:
    """Unit-variance-per-channel Gaussian-blurred noise, [t*h*w, d] float32."""
    t, h, w = grid
    g = torch.randn(t, h, w, d, generator=gen, device=device, dtype=torch.float32)
    for axis, n in enumerate((t, h, w)):
        if n < 2:
            continue
        F = gaussian_filter_matrix(n, sigma, radius, torch.float32).to(device)
        g = torch.movedim(torch.tensordot(F, torch.movedim(g, axis, 0), dims=1), 0, axis)
    g = g.reshape(t * h * w, d)
    std = g.std(dim=0, unbiased=False).clamp_min(1e-12)
    return g / std


def make_qkv(grid, heads: int, d: int, seed: int, batch: int = 1, text_tokens: int = 0,
             dtype=torch.bfloat16, device="cpu"):
    """Q, K, V of shape [batch, heads, L, d] following the recipe above."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    t, h, w = grid
    Lv = t * h * w
    L = Lv + text_tokens
    Q = torch.empty(batch, heads, L, d, dtype=dtype, device=device)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)
    for b in range(batch):
        for hd in range(heads):
            G = smooth_field(grid, d, gen, device)
            n1 = torch.randn(Lv, d, generator=gen, device=device)
            n2 = torch.randn(Lv, d, generator=gen, device=device)
            v = torch.randn(Lv, d, generator=gen, device=device)
            Q[b, hd, :Lv] = (G + 0.5 * n1).to(dtype)
            K[b, hd, :Lv] = (G + 0.5 * n2).to(dtype)
            V[b, hd, :Lv] = v.to(dtype)
            if text_tokens:
                Q[b, hd, Lv:] = torch.randn(text_tokens, d, generator=gen, device=device).to(dtype)
                K[b, hd, Lv:] = torch.randn(text_tokens, d, generator=gen, device=device).to(dtype)
                V[b, hd, Lv:] = torch.randn(text_tokens, d, generator=gen, device=device).to(dtype)
    return Q, K, V


def make_workload(wl: Workload, device="cpu", seed_offset: int = 0):
    """Q, K, V for a named workload (seed_offset gives independent replicas)."""
    return make_qkv(wl.grid, wl.heads, wl.d, wl.seed + seed_offset, wl.batch, wl.text_tokens, wl.dtype, device)


def make_iid(batch: int, heads: int, L: int, d: int, seed: int, dtype=torch.float32, device="cpu",
             scale: float = 1.0):
    """iid N(0, scale^2) Q, K, V [batch, heads, L, d] (edge-case tests)."""
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(int(seed))
    shape = (batch, heads, L, d)
    Q = (scale * torch.randn(shape, generator=gen, device=device)).to(dtype)
    K = (scale * torch.randn(shape, generator=gen, device=device)).to(dtype)
    V = torch.randn(shape, generator=gen, device=device).to(dtype)
    return Q, K, V
