"""Seeded synthetic inputs for the SquareQ W4 linear layer.

This module only draws random tensors: it holds none of the layer's
arithmetic, and both the CUDA path's tests/bench and the CPU oracle take their
inputs from here.  The pages' model weights and activations (FLUX.2 Klein-4B,
Krea-2, LTX-2) are not available, so these tensors stand in for them with the
pages' GEMM shapes (SquareQ README, NVFP4 vs bf16 table: 1536x3072x3072 ...
4480x6144x16384) and the value distributions below.

Shapes: x [M, K] bf16 (bit patterns as uint16), R [N, K] fp32 (the residual
before rotation), lora_up U [N, 32] bf16, lora_down D [K, 32] bf16.

Recipes (numpy PCG64 seeded with the config's seed; draws in blocks of 256
rows; order: x normals, channel scales, R (per row block: normals, then the
outlier uniforms or the chi-square gammas), D, U, hot channel indices):
  "normal"  : x = bf16(z * exp(0.5 * z'_k))   (per-input-channel lognormal
              scale, sigma 0.5); R = N(0, 1/sqrt(K)) with each entry
              independently x8 with probability 0.01 (outliers).
  "student" : x as above; R = Student-t(4) scaled by 1/sqrt(2K) (std 1/sqrt(K)).
  hot_channels (int): that many distinct input channels (indices drawn after
              everything else) are scaled x20 in both x and R.
  U, D      : bf16 N(0, 0.02).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

RANK = 32


@dataclass(frozen=True)
class Config:
    name: str
    M: int
    K: int
    N: int
    seed: int
    dist: str = "normal"
    hot_channels: int = 0


# names give M x N x K (tokens x out x in), the order of the pages' GEMM table
CONFIGS = {
    "tiny_64x256x512": Config("tiny_64x256x512", 64, 512, 256, 0, "normal"),
    "proj_1536x3072x3072": Config("proj_1536x3072x3072", 1536, 3072, 3072, 1, "normal"),
    "qkv_1536x9216x3072": Config("qkv_1536x9216x3072", 1536, 3072, 9216, 2, "normal", 4),
    "large_4480x6144x6144": Config("large_4480x6144x6144", 4480, 6144, 6144, 3, "student"),
    "large_4480x16384x6144": Config("large_4480x16384x6144", 4480, 6144, 16384, 3, "student"),
    "down_4480x6144x16384": Config("down_4480x6144x16384", 4480, 16384, 6144, 4, "student"),
}

# the builder stack: 28 residual weights of the down-projection shape
STACK_COUNT = 28


def stack_seed(i: int) -> int:
    return 4 * 1000 + i


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even (torch)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


_CHUNK = 256  # rows drawn per call; part of the recipe (fixes the stream order)


def _residual(rng: np.random.Generator, N: int, K: int, dist: str) -> np.ndarray:
    R = np.empty((N, K), np.float32)
    if dist == "zero":
        R[:] = 0.0
        return R
    z = np.empty((_CHUNK, K), np.float32)
    u = np.empty((_CHUNK, K), np.float32)
    for r0 in range(0, N, _CHUNK):
        rows = min(_CHUNK, N - r0)
        zc, uc, out = z[:rows], u[:rows], R[r0:r0 + rows]
        rng.standard_normal(out=zc, dtype=np.float32)
        if dist == "normal":
            rng.random(out=uc, dtype=np.float32)
            np.multiply(zc, np.float32(1.0 / np.sqrt(K)), out=out)
            out[uc < np.float32(0.01)] *= np.float32(8.0)
        elif dist == "student":
            rng.standard_gamma(2.0, out=uc, dtype=np.float32)   # chi^2(4) / 4 = Gamma(2) / 2
            np.multiply(uc, np.float32(0.5), out=uc)
            np.sqrt(uc, out=uc)
            np.divide(zc, uc, out=out)
            np.multiply(out, np.float32(1.0 / np.sqrt(2.0 * K)), out=out)
        else:
            raise ValueError(dist)
    return R


def make_inputs(M: int, K: int, N: int, seed: int, dist: str = "normal", hot_channels: int = 0):
    """Return dict(x, R, U, D) for one layer (see the module docstring)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    xf = np.empty((M, K), np.float32)
    for r0 in range(0, M, _CHUNK):
        rng.standard_normal(out=xf[r0:r0 + _CHUNK], dtype=np.float32)
    ch = np.exp(np.float32(0.5) * rng.standard_normal(K, dtype=np.float32)).astype(np.float32)
    R = _residual(rng, N, K, dist)
    D = rng.standard_normal((K, RANK), dtype=np.float32) * np.float32(0.02)
    U = rng.standard_normal((N, RANK), dtype=np.float32) * np.float32(0.02)
    np.multiply(xf, ch[None, :], out=xf)
    if hot_channels:
        hot = rng.choice(K, size=hot_channels, replace=False)
        xf[:, hot] *= np.float32(20.0)
        R[:, hot] *= np.float32(20.0)
    return {
        "x": to_bf16_bits(xf),
        "R": R,
        "U": to_bf16_bits(U),
        "D": to_bf16_bits(D),
    }


def make_config(name: str):
    c = CONFIGS[name]
    return make_inputs(c.M, c.K, c.N, c.seed, c.dist, c.hot_channels)


def make_stack_residual(i: int, N: int = 6144, K: int = 16384) -> np.ndarray:
    """Residual i of the 28-weight builder stack (down-projection shape, Student-t)."""
    rng = np.random.Generator(np.random.PCG64(stack_seed(i)))
    return _residual(rng, N, K, "student")


def make_stack_residual_device(i: int, out, N: int = 6144, K: int = 16384):
    """The same distribution drawn on a CUDA device into `out` (fp32 [N, K]) with torch's seeded
    generator (seed stack_seed(i)): z / sqrt(Gamma(2) / 2) / sqrt(2 K), a Student-t(4) scaled to
    std 1/sqrt(K).  A different stream from make_stack_residual, for timing only (numpy takes
    seconds per weight)."""
    g = torch.Generator(device=out.device).manual_seed(stack_seed(i))
    torch.randn((N, K), generator=g, device=out.device, out=out)
    chi = torch._standard_gamma(torch.full((N, K), 2.0, device=out.device), generator=g)
    out.div_(chi.mul_(0.5).sqrt_()).mul_(float(1.0 / np.sqrt(2.0 * K)))
    return out
