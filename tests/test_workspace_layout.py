"""Exact forward workspace sizes (host-side layout arithmetic of sq_api.cu, no GPU).

The layout is a 256-byte header, then each region starting on a 1024-byte boundary, and the
total rounded up to 1024 bytes:
  NVFP4:     activation codes M K / 2, tiled scales sq_sf_bytes(M, K);
  int4/int8: bf16(H x) M K 2, the W ring R 256 K 2 with R = min(ceil(N / 256),
             ceil(74 / ceil(M / 256)) + 2), and its 2 R u32 counters;
  then t's partial tiles parts M 32 4, [t_hi | t_lo] M 64 2, [U | U] N 64 2, and, for int8,
  the rank-16 factors widened to rank 32: K 32 2 and N 32 2.
parts = act_t_parts(M, K) = min(16, K / 256, max(1, 148 // ceil(M / 128))).
"""
import math

import pytest

import bit_quantized_frozen_b200 as sq


def up(v, a=1024):
    return (v + a - 1) // a * a


def t_parts(M, K):
    tiles = math.ceil(M / 128)
    return min(16, K // 256, max(1, 148 // tiles))


def ring_slots(M, N):
    return min(math.ceil(N / 256), math.ceil(74 / math.ceil(M / 256)) + 2)


def expected(fmt, M, N, K):
    regions = []
    if fmt == "nvfp4":
        regions += [M * K // 2, sq.sq_sf_bytes(M, K)]
    else:
        R = ring_slots(M, N)
        regions += [M * K * 2, R * 256 * K * 2, 2 * R * 4]
    regions += [t_parts(M, K) * M * 32 * 4, M * 64 * 2, N * 64 * 2]
    if fmt == "int8":
        regions += [K * 32 * 2, N * 32 * 2]
    off = 256
    for b in regions:
        off = up(off) + b
    return up(off)


SHAPES = [(1, 128, 256), (64, 256, 512), (127, 384, 512), (300, 1280, 512), (1536, 3072, 3072),
          (1536, 9216, 3072), (2560, 4096, 512), (4480, 16384, 6144), (4480, 6144, 16384), (9600, 512, 256)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "int8"])
def test_forward_workspace_bytes(fmt, M, N, K):
    op = {"nvfp4": sq.SQ_OP_LINEAR_FWD_NVFP4, "int4": sq.SQ_OP_LINEAR_FWD_INT4,
          "int8": sq.SQ_OP_LINEAR_FWD_INT8}[fmt]
    assert sq.sq_workspace_bytes(op, M, N, K) == expected(fmt, M, N, K)


def test_the_ring_does_not_grow_with_n_beyond_the_tiles_in_flight():
    # at M = 4480 the ring has 7 slots for any N of 7 or more W tiles
    base = sq.sq_workspace_bytes(sq.SQ_OP_LINEAR_FWD_INT4, 4480, 7 * 256, 6144)
    big = sq.sq_workspace_bytes(sq.SQ_OP_LINEAR_FWD_INT4, 4480, 64 * 256, 6144)
    assert big - base == up(64 * 256 * 128) - up(7 * 256 * 128)       # only [U | U] grows
