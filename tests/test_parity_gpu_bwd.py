"""Backward of the input (SquareQ README, "End-to-end": the backward rebuilds bf16 W
from the same payload and runs the normal bf16 GEMM) through the C ABI against the
CPU oracle: the transposed reconstruct W^T bit for bit (every payload format, with
and without the low-rank term), and dx = dy W within max|dx - dx_oracle| /
max|dx_oracle| <= 2e-3, the oracle evaluating dy W in fp64 on the same bf16
operands.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from sqcase import FWD_TOL, bf16_dev, bits16, first_mismatch, host, norm_err, to_dev

pytestmark = pytest.mark.gpu

FMTS = ["nvfp4", "int4", "int4_g64", "int8"]


@pytest.fixture(scope="module")
def sq():
    import bit_quantized_frozen_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


def weight_and_oracle_W(sq, d, fmt, lora=True):
    """GPU weight of the given format and the oracle's bf16 reconstruct of the same payload."""
    N, K = d["R"].shape
    R = to_dev(d["R"])
    if fmt == "int8":
        U, D = np.ascontiguousarray(d["U"][:, :16]), np.ascontiguousarray(d["D"][:, :16])
    else:
        U, D = d["U"], d["D"]
    Ud, Dd = (bf16_dev(U), bf16_dev(D)) if lora else (None, None)
    if fmt == "nvfp4":
        w = sq.build_nvfp4(R, Ud, Dd)
        c, s, g = oracle.build_nvfp4(d["R"])
        f = oracle.FMT_NVFP4
    elif fmt == "int8":
        w = sq.build_int8(R, Ud, Dd)
        c, s, _ = oracle.build_int8(d["R"])
        g, f = 0.0, oracle.FMT_INT8_ROW
    else:
        grp = 64 if fmt == "int4_g64" else 32
        w = sq.build_int4(R, Ud, Dd, group=grp)
        c, s, _ = oracle.build_int4(d["R"], group=grp)
        g, f = 0.0, oracle.FMT_INT4_G64 if grp == 64 else oracle.FMT_INT4
    Wo = oracle.reconstruct_bf16(f, c, s, g, U, D, N, K, residual_only=not lora)
    return w, Wo


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("lora", [True, False], ids=["lowrank", "residual"])
def test_reconstruct_transposed(sq, fmt, lora):
    d = si.make_inputs(8, 768, 384, 61)
    w, Wo = weight_and_oracle_W(sq, d, fmt, lora)
    Wt = sq.reconstruct_bf16(w, residual_only=not lora, transposed=True)
    torch.cuda.synchronize()
    assert tuple(Wt.shape) == (768, 384)
    got = bits16(Wt)
    want = np.ascontiguousarray(Wo.T)
    assert np.array_equal(got, want), first_mismatch(got, want)


def check_dx(sq, d, fmt, M, rows=None, seed=62):
    w, Wo = weight_and_oracle_W(sq, d, fmt)
    N = d["R"].shape[0]
    rng = np.random.default_rng(seed)
    dy = si.to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    dx = sq.linear_bwd_dx(w, bf16_dev(dy))
    torch.cuda.synchronize()
    rows = np.arange(M, dtype=np.int64) if rows is None else rows
    want = oracle.linear_bwd_dx(dy, Wo, rows)
    got = host(dx)[rows]
    assert np.all(np.isfinite(got))
    err = norm_err(got, want)
    assert err <= FWD_TOL, f"normalised error {err:.3e}"


@pytest.mark.parametrize("fmt", FMTS)
def test_bwd_dx_small(sq, fmt):
    check_dx(sq, si.make_inputs(8, 512, 256, 63), fmt, M=200)


@pytest.mark.parametrize("shape", [(1, 256, 128), (129, 768, 384), (64, 1280, 640)])
def test_bwd_dx_edge_shapes(sq, shape):
    M, K, N = shape
    check_dx(sq, si.make_inputs(8, K, N, 64 + M), "nvfp4", M=M)


def test_bwd_dx_proj_sampled(sq):
    d = si.make_config("proj_1536x3072x3072")
    rng = np.random.default_rng(65)
    rows = np.unique(np.concatenate([[0, 1535], rng.choice(1536, 30, replace=False)])).astype(np.int64)
    check_dx(sq, d, "nvfp4", M=1536, rows=rows)


@pytest.mark.slow
def test_bwd_bench_shape_sampled(sq):
    """The bench workload 4480 x 16384 x 6144 (NVFP4 payload, as the bench times it): W^T bit
    for bit on sampled rows, dx within tolerance on sampled rows."""
    d = si.make_config("large_4480x16384x6144")
    M = d["x"].shape[0]
    w, Wo = weight_and_oracle_W(sq, d, "nvfp4")
    Wt = sq.reconstruct_bf16(w, transposed=True)
    rng = np.random.default_rng(66)
    dy = si.to_bf16_bits(rng.standard_normal((M, Wo.shape[0])).astype(np.float32))
    dx = sq.linear_bwd_dx(w, bf16_dev(dy))
    torch.cuda.synchronize()
    krows = np.unique(np.concatenate([[0, Wo.shape[1] - 1], rng.choice(Wo.shape[1], 24, replace=False)]))
    got = bits16(Wt)[krows]
    want = np.ascontiguousarray(Wo[:, krows].T)
    assert np.array_equal(got, want), first_mismatch(got, want)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 6, replace=False)])).astype(np.int64)
    err = norm_err(host(dx)[rows], oracle.linear_bwd_dx(dy, Wo, rows))
    assert err <= FWD_TOL, f"normalised error {err:.3e}"
