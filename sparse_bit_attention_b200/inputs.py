"""Seeded synthetic inputs shaped like the Wan2.1 self-attention workloads.

This module only draws random tensors; it holds none of the attention method's arithmetic,
so both the CUDA path's tests and the CPU oracle's tests can take their inputs from it.

Recipe (all draws from one ``torch.Generator`` on the CPU, in float32, then rounded to
bf16):
* random workloads: Q, K, V ~ N(0, 1) drawn in that order, shape [B, H, N, 128];
* ``tiny``: as above, then one offset per (head, channel) ~ N(0, variance 2) added to K,
  so that K has a non-zero channel mean for the smoothing step to remove;
* ``locality_14b_720p``: on the 21 x 45 x 80 (t, y, x) latent grid, token index
  n = (t * 45 + y) * 80 + x. One white-noise field per (head, channel) is filtered by a
  separable Gaussian (sigma 3 tokens, radius 12, normalized weights, reflected borders) and
  rescaled to unit variance, giving F. Then Q = F + 0.3 eps_q and K = F + 0.3 eps_k share F,
  and V ~ N(0, 1).
"""
from __future__ import annotations

import dataclasses
import math

import torch

HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    seed: int
    topk_ratios: tuple
    kind: str = "normal"            # "normal" | "offset" | "locality"
    grid: tuple | None = None       # (T, Y, X) for the locality field
    description: str = ""


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 1024, 0, (0.1, 1.0), kind="offset",
                     description="B1 H2 N1024 d128, 16x16 blocks, K with channel offsets"),
    "wan21_1p3b_480p": Workload("wan21_1p3b_480p", 1, 12, 32760, 1, (0.1,),
                                grid=(21, 30, 52),
                                description="Wan2.1-1.3B-480P self-attention shape"),
    "wan21_14b_480p": Workload("wan21_14b_480p", 1, 40, 32760, 2, (0.1,),
                               grid=(21, 30, 52),
                               description="Wan2.1-14B-480P self-attention shape"),
    "wan21_14b_720p": Workload("wan21_14b_720p", 1, 40, 75600, 3, (0.1,),
                               grid=(21, 45, 80),
                               description="Wan2.1-14B-720P self-attention shape"),
    "locality_14b_720p": Workload("locality_14b_720p", 1, 40, 75600, 4, (0.05, 0.1, 0.15),
                                  kind="locality", grid=(21, 45, 80),
                                  description="smoothed-field Q/K on the 14B-720P grid"),
}


def _gaussian_taps(sigma: float, radius: int) -> torch.Tensor:
    x = torch.arange(-radius, radius + 1, dtype=torch.float64)
    w = torch.exp(-0.5 * (x / sigma) ** 2)
    return (w / w.sum()).to(torch.float32)


def _smooth_fields(noise: torch.Tensor, sigma: float = 3.0, radius: int = 12) -> torch.Tensor:
    """Separable Gaussian filter over the last three axes of [F, T, Y, X], reflected borders,
    then each field rescaled to unit variance."""
    taps = _gaussian_taps(sigma, radius)
    f = noise
    for axis in (1, 2, 3):
        f = f.movedim(axis, -1)
        shape = f.shape
        flat = f.reshape(-1, 1, shape[-1])
        flat = torch.nn.functional.pad(flat, (radius, radius), mode="reflect")
        flat = torch.nn.functional.conv1d(flat, taps.view(1, 1, -1))
        f = flat.reshape(shape).movedim(-1, axis)
    std = f.flatten(1).std(dim=1, unbiased=False).clamp_min(1e-12)
    return f / std.view(-1, 1, 1, 1)


def make_qkv(name: str, n_tokens: int | None = None, heads: int | None = None):
    """Q, K, V for a named workload as bf16 CPU tensors [B, H, N, 128].

    ``n_tokens`` / ``heads`` override N and H of the random workloads (used for small parity
    cases with the same distribution); the draws are then of the overridden shape."""
    w = WORKLOADS[name]
    B = w.B
    H = heads if heads is not None else w.H
    N = n_tokens if n_tokens is not None else w.N
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (B, H, N, HEAD_DIM)
    if w.kind == "locality":
        T, Y, X = w.grid
        assert N == T * Y * X, "the locality field lives on the full latent grid"
        noise = torch.randn((B * H * HEAD_DIM, T, Y, X), generator=g, dtype=torch.float32)
        fields = torch.empty_like(noise)
        chunk = 512
        for s in range(0, noise.shape[0], chunk):
            fields[s:s + chunk] = _smooth_fields(noise[s:s + chunk])
        del noise
        F = fields.view(B, H, HEAD_DIM, N).transpose(2, 3)   # n = (t*Y + y)*X + x
        eq = torch.randn(shape, generator=g, dtype=torch.float32)
        q = (F + 0.3 * eq).to(torch.bfloat16)
        del eq
        ek = torch.randn(shape, generator=g, dtype=torch.float32)
        k = (F + 0.3 * ek).to(torch.bfloat16)
        del ek, F, fields
        v = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
        return q.contiguous(), k.contiguous(), v.contiguous()
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if w.kind == "offset":
        off = torch.randn((B, H, 1, HEAD_DIM), generator=g, dtype=torch.float32) * math.sqrt(2.0)
        k = k + off
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_random(B: int, H: int, N: int, seed: int, k_offset_std: float = 0.0,
                scale: float = 1.0, qk_scale: float = 1.0, v_mean_std: float = 0.0):
    """Q, K, V ~ N(0, scale^2) bf16 [B, H, N, 128]; optional per-(b,h,channel) K offset
    ~ N(0, k_offset_std^2); Q and K further multiplied by ``qk_scale`` (large logits); optional
    per-(b,h,channel) V mean ~ N(0, v_mean_std^2), drawn after the K offset."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, H, N, HEAD_DIM)
    q = torch.randn(shape, generator=g, dtype=torch.float32) * scale
    k = torch.randn(shape, generator=g, dtype=torch.float32) * scale
    v = torch.randn(shape, generator=g, dtype=torch.float32) * scale
    if k_offset_std:
        k = k + torch.randn((B, H, 1, HEAD_DIM), generator=g, dtype=torch.float32) * k_offset_std
    if v_mean_std:
        v = v + torch.randn((B, H, 1, HEAD_DIM), generator=g, dtype=torch.float32) * v_mean_std
    if qk_scale != 1.0:
        q, k = q * qk_scale, k * qk_scale
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def as_float64(t: torch.Tensor):
    """bf16 tensor -> float64 numpy array of the same values (exact)."""
    return t.to(torch.float64).numpy()
