"""Seeded synthetic inputs shaped like video-DiT attention layers.

This module only draws inputs; it holds none of the attention method's
arithmetic, and both the CUDA path and the float64 oracle consume what it
returns. Everything is generated with torch from explicit seeds, then rounded
to bf16 (round-to-nearest-even) so both sides see identical bits.

Generators:

* ``gaussian_with_sinks``  N(0, 1) Q/K/V plus key "sink" tokens whose norm is 8x
  the mean key norm, pointing along the head's mean query (small parity case).
* ``smoothed_field``       a spatio-temporally smoothed Gaussian field on a
  t x h x w latent grid (Wan2.1-style video tokens, flattened t-major) with
  K correlated to Q so attention is local, V independent, and 4 sink keys.
* ``mixed_rows``           the smoothed field with alternating q-blocks made
  near-uniform (queries scaled by 0.1) or skewed (+6 logit on kv-block 0).
"""

from __future__ import annotations

import math

import torch

# latent grids (t, h, w) of the Wan2.1 shapes: 21x30x52 = 32760 (1.3B, 480p),
# 21x45x80 = 75600 (14B, 720p), and the sweep's extra lengths
GRIDS = {
    32760: (21, 30, 52),
    75600: (21, 45, 80),
    8192: (8, 32, 32),
    65536: (16, 64, 64),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _seed(*parts: int) -> int:
    s = 0x9E3779B97F4A7C15
    for p in parts:
        s = (s * 6364136223846793005 + int(p) + 1442695040888963407) & 0xFFFFFFFFFFFFFFFF
    return s >> 1


def _add_sinks(q: torch.Tensor, k: torch.Tensor, n_sinks: int) -> torch.Tensor:
    """k[..., :n_sinks, :] <- 8 * mean key norm * (mean query direction)."""
    qbar = q.mean(dim=-2, keepdim=True)
    qhat = qbar / qbar.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    knorm = k.norm(dim=-1).mean(dim=-1, keepdim=True)[..., None]
    k = k.clone()
    k[..., :n_sinks, :] = (8.0 * knorm * qhat).expand(*k.shape[:-2], n_sinks, k.shape[-1])
    return k


def gaussian_with_sinks(B=1, H=2, N=512, d=64, seed=0, n_sinks=2, device="cpu"):
    """Q, K, V ~ N(0, 1) (bf16) with ``n_sinks`` sink keys per head."""
    g = _gen(_seed(1, seed))
    q = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    k = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    k = _add_sinks(q, k, n_sinks)
    return tuple(x.to(torch.bfloat16).to(device) for x in (q, k, v))


def normal_like(shape, seed, device="cpu"):
    """N(0, 1) bf16 tensor (used for the output gradient dO)."""
    g = _gen(_seed(2, seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16).to(device)


def _gauss_kernel(sigma: float) -> torch.Tensor:
    r = max(1, int(math.ceil(3.0 * sigma)))
    x = torch.arange(-r, r + 1, dtype=torch.float32)
    w = torch.exp(-0.5 * (x / sigma) ** 2)
    return w / w.sum()


def _blur_axis(x: torch.Tensor, axis: int, sigma: float) -> torch.Tensor:
    # x: [C, T, Hg, Wg]; separable 1-D Gaussian along `axis` (1..3), reflect padding
    w = _gauss_kernel(sigma).to(x.device)
    r = (w.numel() - 1) // 2
    xm = x.movedim(axis, -1)
    shp = xm.shape
    flat = xm.reshape(-1, 1, shp[-1])
    flat = torch.nn.functional.pad(flat, (r, r), mode="reflect")
    flat = torch.nn.functional.conv1d(flat, w.view(1, 1, -1))
    return flat.reshape(shp).movedim(-1, axis)


def _field(grid, d, seed, device):
    """One smoothed field [N, d]: white noise, blur sigma=(1, 1.5, 1.5) cells, unit variance."""
    t, h, w = grid
    g = _gen(seed)
    z = torch.randn(d, t, h, w, generator=g, dtype=torch.float32).to(device)
    for axis, sigma in ((1, 1.0), (2, 1.5), (3, 1.5)):
        z = _blur_axis(z, axis, sigma)
    z = z.reshape(d, -1)
    z = (z - z.mean(dim=1, keepdim=True)) / z.std(dim=1, keepdim=True).clamp_min(1e-12)
    return z.t().contiguous()        # [N, d], t-major token order


def smoothed_field(B=1, H=12, N=32760, d=128, seed=0, n_sinks=4, device="cpu", grid=None):
    """Wan2.1-shaped Q/K/V (bf16): K = 0.5 Q + sqrt(0.75) noise field; V independent."""
    grid = grid or GRIDS[N]
    assert grid[0] * grid[1] * grid[2] == N
    q = torch.empty(B, H, N, d, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    for b in range(B):
        for h in range(H):
            fq = _field(grid, d, _seed(10, seed, b, h, 0), device)
            fk = _field(grid, d, _seed(10, seed, b, h, 1), device)
            fv = _field(grid, d, _seed(10, seed, b, h, 2), device)
            q[b, h] = fq
            k[b, h] = 0.5 * fq + math.sqrt(0.75) * fk
            v[b, h] = fv
    k = _add_sinks(q, k, n_sinks)
    return tuple(x.to(torch.bfloat16) for x in (q, k, v))


def mixed_rows(B=1, H=12, N=32760, d=128, seed=0, bq=128, bkv=64, device="cpu", grid=None):
    """Smoothed field with even q-blocks near-uniform and odd q-blocks skewed.

    Even q-blocks: queries scaled by 0.1 (logits shrink tenfold).
    Odd q-blocks: a shared vector s (|s| = sqrt(d)) is added to every key of
    kv-block 0 and 6*s_hat to the queries, so kv-block 0 gains a +6 logit.
    """
    q, k, v = smoothed_field(B, H, N, d, seed, n_sinks=0, device=device, grid=grid)
    q = q.float(); k = k.float()
    g = _gen(_seed(20, seed))
    s = torch.randn(B, H, 1, d, generator=g).to(device)
    s_hat = s / s.norm(dim=-1, keepdim=True)
    s = s_hat * math.sqrt(d)
    blk = torch.arange(N, device=device) // bq
    even = (blk % 2 == 0).view(1, 1, N, 1)
    q = torch.where(even, 0.1 * q, q + 6.0 * s_hat)
    k[..., :min(bkv, N), :] += s
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v
