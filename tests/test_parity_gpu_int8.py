"""int8 per-row residual with the rank-16 low-rank branch (SquareQ README, "v3.1 --
int8-residual mode") through the C ABI against the CPU oracle on the same seeded
inputs.

The builder's int8 codes, fp32 row scales and winning fraction indices are compared
bit for bit, the bf16 reconstruct bit for bit, the "dequant-first" forward within
max|dy| / max|y| <= 2e-3 of the oracle's fp64 result on the same operands.  The
rank-16 factors are the first 16 columns of each config's rank-32 factors.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from sqcase import FWD_TOL, bf16_dev, bits16, first_mismatch, host, norm_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    import bit_quantized_frozen_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


@functools.lru_cache(maxsize=1)
def inputs(name):
    return si.make_config(name)


def rank16(d):
    return np.ascontiguousarray(d["U"][:, :16]), np.ascontiguousarray(d["D"][:, :16])


def sample_rows(n, count, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(count, n), replace=False)]))
    return rows.astype(np.int64)


def check_build(sq, R, rows=None):
    w = sq.build_int8(to_dev(R))
    torch.cuda.synchronize()
    assert w.fmt == sq.SQ_FMT_INT8_ROW
    sel = slice(None) if rows is None else rows
    oc, os_, of = oracle.build_int8(R[sel])
    codes, scales, frac = host(w.codes)[sel], host(w.scales)[sel], host(w.frac_idx)[sel]
    assert np.array_equal(codes, oc), first_mismatch(codes, oc)
    assert np.array_equal(scales.view(np.uint32), os_.view(np.uint32)), first_mismatch(scales, os_)
    assert np.array_equal(frac, of), first_mismatch(frac, of)


@pytest.mark.parametrize("name", ["tiny_64x256x512", "proj_1536x3072x3072"])
def test_build_int8(sq, name):
    check_build(sq, inputs(name)["R"])


def test_build_int8_sampled_qkv(sq):
    R = inputs("qkv_1536x9216x3072")["R"]
    check_build(sq, R, sample_rows(R.shape[0], 96, 51))


def test_build_int8_block_counts_and_special_rows(sq):
    """Rows of 1, 3, 33 and 64 Hadamard blocks (partial 8-lane groups in the last warp,
    several blocks per group), an all-zero row and a row with one huge outlier."""
    for K in (256, 768, 8448, 16384):
        d = si.make_inputs(4, K, 128, 52 + K)
        R = d["R"].copy()
        R[5, :] = 0.0
        R[9, K // 3] = 1e3
        check_build(sq, R)


def check_fwd(sq, d, rows=None, lora=True):
    M, K = d["x"].shape
    N = d["R"].shape[0]
    U16, D16 = rank16(d)
    U = bf16_dev(U16) if lora else None
    D = bf16_dev(D16) if lora else None
    w = sq.build_int8(to_dev(d["R"]), U, D)
    y = sq.linear_fwd(w, bf16_dev(d["x"]))
    torch.cuda.synchronize()
    rows = np.arange(M, dtype=np.int64) if rows is None else rows
    codes, scales, _ = oracle.build_int8(d["R"])
    t = oracle.lowrank_input(d["x"], D16) if lora else None
    xr = oracle.rotate_rows_bf16(d["x"])
    y_ref = oracle.linear_fwd_int8(xr, codes, scales, t, U16 if lora else None, M, N, K, rows)
    y_gpu = host(y)[rows]
    assert np.all(np.isfinite(y_gpu))
    err = norm_err(y_gpu, y_ref)
    assert err <= FWD_TOL, f"normalised error {err:.3e}"


def test_linear_fwd_int8_tiny(sq):
    check_fwd(sq, inputs("tiny_64x256x512"))


def test_linear_fwd_int8_proj_sampled(sq):
    d = inputs("proj_1536x3072x3072")
    check_fwd(sq, d, sample_rows(d["x"].shape[0], 32, 53))


@pytest.mark.parametrize("shape", [(1, 256, 128), (127, 512, 384), (300, 1280, 512)])
def test_linear_fwd_int8_edge_shapes(sq, shape):
    M, K, N = shape
    check_fwd(sq, si.make_inputs(M, K, N, 300 + M))


def test_linear_fwd_int8_ring_slot_reuse(sq):
    """M = 2560 (10 M tiles) and N = 4096 (16 W tiles): the GEMM's W ring has
    ceil(74 / 10) + 2 = 10 slots, so six slots take a second W tile once its ten clusters are
    done with the first.  Sampled rows, the last M tile's among them."""
    d = si.make_inputs(2560, 512, 4096, 355)
    rows = np.unique(np.concatenate([sample_rows(2560, 40, 56), np.arange(2552, 2560)])).astype(np.int64)
    check_fwd(sq, d, rows)


def test_linear_fwd_int8_without_lowrank(sq):
    check_fwd(sq, si.make_inputs(150, 512, 256, 54), lora=False)


def check_reconstruct(sq, d, residual_only=False, rows=None):
    N, K = d["R"].shape
    U16, D16 = rank16(d)
    w = sq.build_int8(to_dev(d["R"]), bf16_dev(U16), bf16_dev(D16))
    W = sq.reconstruct_bf16(w, residual_only=residual_only)
    torch.cuda.synchronize()
    sel = slice(None) if rows is None else rows
    c, s, _ = oracle.build_int8(d["R"][sel])
    Wo = oracle.reconstruct_bf16(oracle.FMT_INT8_ROW, c, s, 0.0, U16[sel], D16, len(c), K, residual_only)
    Wg = bits16(W)[sel]
    assert np.array_equal(Wg, Wo), first_mismatch(Wg, Wo)


@pytest.mark.parametrize("name", ["tiny_64x256x512", "proj_1536x3072x3072"])
def test_reconstruct_int8(sq, name):
    check_reconstruct(sq, inputs(name))


def test_reconstruct_int8_residual_only_ragged(sq):
    check_reconstruct(sq, si.make_inputs(8, 768, 384, 55), residual_only=True)


@pytest.mark.slow
def test_large_int8_sampled(sq):
    d = inputs("down_4480x6144x16384")
    N = d["R"].shape[0]
    check_build(sq, d["R"], sample_rows(N, 24, 56))
    check_reconstruct(sq, d, rows=sample_rows(N, 12, 57))
    check_fwd(sq, d, sample_rows(d["x"].shape[0], 6, 58))
