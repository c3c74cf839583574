"""Test helpers: run one layer through the CUDA path (via the C ABI binding)
and through the CPU oracle on the same seeded inputs, and compare.

Comparison rules (from the layer's contract in include/sq.h):
  - codes, scales, scale-fraction indices, tiled scale bytes, g_w / g_x:
    bit-exact;
  - bf16 reconstruct: bit-exact;
  - forward outputs: max|y_gpu - y_oracle| / max|y_oracle| <= 2e-3, the oracle
    evaluating the same quantised operands in fp64.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth_inputs as si

FWD_TOL = 2e-3


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return to_dev(bits.view(np.int16), None).view(torch.bfloat16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def norm_err(y_gpu: np.ndarray, y_ref: np.ndarray) -> float:
    denom = float(np.abs(y_ref).max())
    diff = float(np.abs(y_gpu.astype(np.float64) - y_ref).max())
    return diff / denom if denom > 0 else diff


def sf_rows_equal(sf_a: np.ndarray, sf_b: np.ndarray, rows, K: int) -> bool:
    """Compare the tiled scale bytes of the given rows."""
    C = K // 16
    r = np.asarray(rows, np.int64)[:, None]
    c = np.arange(C, dtype=np.int64)[None, :]
    off = ((r // 128) * (C // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)
    return np.array_equal(sf_a[off], sf_b[off])


def first_mismatch(a: np.ndarray, b: np.ndarray) -> str:
    idx = np.argwhere(a != b)
    if len(idx) == 0:
        return "equal"
    i = tuple(idx[0])
    return f"{len(idx)} mismatches, first at {i}: gpu={a[i]} oracle={b[i]}"
