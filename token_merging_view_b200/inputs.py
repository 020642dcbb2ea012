"""Seeded synthetic Q/K/V shaped like a VGGT global-attention layer.

This module holds no part of the merging method: it only makes inputs.  Both
the CUDA path and the fp64 oracle consume the exact bytes it produces (the
oracle through a host copy), so the random stream never has to be reproduced
on the other side.

Recipe (one tensor X in {Q, K, V}, per head):

1. ``gen = torch.Generator(device).manual_seed(seed)``.
2. Per-frame integer grid shifts (dy_t, dx_t), each uniform in
   [-max_shift, max_shift] (0 disables them); shared by all heads and by Q, K, V.
3. For each of Q, K, V and each head: Z ~ N(0, 1) on a (G + 2m) x (G + 2m) x d
   grid, G the patch-grid side, m = max_shift the margin.
4. Separable Gaussian blur of each channel, sigma = 1.5 patches, radius 6,
   weights summing to 1, mirror ("reflect") boundary.
5. Divide by sqrt(sum of the squared 2-D weights), so the field has unit
   variance (without it a sigma = 1.5 blur leaves a std near 0.19 and the noise
   would swamp the field).
6. F(t, p = (py, px)) = blurred[py + m + dy_t, px + m + dx_t]  (raster p).
7. e ~ N(0, 1) of shape [h, T, P, d];  X = F + noise_sigma * e.
8. Cast to the storage dtype (bf16 with round-to-nearest-even, or fp32).

The layout is [h, N = T*P, d] row-major, token n = t*P + p.
"""
from __future__ import annotations

import math

import torch


def _gauss_weights(sigma: float, radius: int) -> torch.Tensor:
    x = torch.arange(-radius, radius + 1, dtype=torch.float64)
    w = torch.exp(-0.5 * (x / sigma) ** 2)
    return w / w.sum()


def _blur_field(z: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    """z: [B, S, S, d] -> separable blur over the two grid axes, mirror boundary."""
    B, S, S2, d = z.shape
    r = (w.numel() - 1) // 2
    k = w.to(z.dtype).to(z.device)
    # rows: move the blurred axis last and run a 1-D convolution per channel
    x = z.permute(0, 1, 3, 2).reshape(B * S * d, 1, S2)  # blur along px
    x = torch.nn.functional.pad(x, (r, r), mode="reflect")
    x = torch.nn.functional.conv1d(x, k.view(1, 1, -1))
    x = x.reshape(B, S, d, S2).permute(0, 3, 2, 1)  # [B, px, d, py]
    x = x.reshape(B * S2 * d, 1, S)
    x = torch.nn.functional.pad(x, (r, r), mode="reflect")
    x = torch.nn.functional.conv1d(x, k.view(1, 1, -1))
    x = x.reshape(B, S2, d, S).permute(0, 3, 1, 2)  # [B, py, px, d]
    return x.contiguous()


def make_qkv(
    *,
    T: int,
    grid: int,
    h: int,
    d: int,
    seed: int,
    noise_sigma: float = 0.3,
    max_shift: int = 2,
    dtype: torch.dtype = torch.bfloat16,
    device: str | torch.device = "cpu",
    blur_sigma: float = 1.5,
    blur_radius: int = 6,
):
    """Return (Q, K, V), each [h, T*grid*grid, d] in ``dtype`` on ``device``."""
    device = torch.device(device)
    gen = torch.Generator(device=device).manual_seed(seed)
    P = grid * grid
    m = max_shift
    if m > 0:
        shifts = torch.randint(-m, m + 1, (T, 2), generator=gen, device=device)
    else:
        shifts = torch.zeros((T, 2), dtype=torch.int64, device=device)
    w = _gauss_weights(blur_sigma, blur_radius)
    norm = math.sqrt(float((w[:, None] * w[None, :]).pow(2).sum()))
    S = grid + 2 * m
    py = torch.arange(grid, device=device).view(1, grid, 1)
    px = torch.arange(grid, device=device).view(1, 1, grid)
    rows = (py + m + shifts[:, 0].view(T, 1, 1)).expand(T, grid, grid).reshape(T, P)
    cols = (px + m + shifts[:, 1].view(T, 1, 1)).expand(T, grid, grid).reshape(T, P)
    out = []
    for _ in range(3):  # Q, K, V
        z = torch.randn((h, S, S, d), generator=gen, device=device, dtype=torch.float32)
        f = _blur_field(z, w) / norm  # [h, S, S, d]
        field = f[:, rows, cols, :]  # [h, T, P, d]
        e = torch.randn((h, T, P, d), generator=gen, device=device, dtype=torch.float32)
        x = field + noise_sigma * e
        out.append(x.reshape(h, T * P, d).to(dtype).contiguous())
        del z, f, field, e, x
    return tuple(out)


def make_score(*, T: int, grid: int, seed: int, blur_sigma: float = 1.5, blur_radius: int = 6,
               device: str | torch.device = "cpu") -> torch.Tensor:
    """A seeded stand-in for a per-token importance map, fp32 [T, grid*grid]:
    per frame an N(0, 1) field on the patch grid, blurred like the Q/K/V
    fields (so neighbouring patches score alike, as edges and flat regions
    do in an image).  Holds no part of any method: inputs only."""
    device = torch.device(device)
    gen = torch.Generator(device=device).manual_seed(seed)
    z = torch.randn((T, grid, grid, 1), generator=gen, device=device, dtype=torch.float64)
    radius = min(blur_radius, grid - 1)                 # a mirror pad needs radius < grid
    f = _blur_field(z, _gauss_weights(blur_sigma, radius).to(device)) if radius > 0 else z
    return f.reshape(T, grid * grid).float()
