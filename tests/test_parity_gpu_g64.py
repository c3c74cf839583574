"""int4 group-64 (SquareQ README, "Residual codecs" paragraph: groups of 32 or 64)
through the C ABI against the CPU oracle on the same seeded inputs.

The builder's codes, fp16 scales and winning fraction indices are compared bit
for bit, the bf16 reconstruct bit for bit, the "dequant-first" forward within
max|dy| / max|y| <= 2e-3 of the oracle's fp64 result on the same operands.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from sqcase import FWD_TOL, bf16_dev, bits16, first_mismatch, host, norm_err, to_dev

pytestmark = pytest.mark.gpu

G = 64


@pytest.fixture(scope="module")
def sq():
    import bit_quantized_frozen_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


@functools.lru_cache(maxsize=1)
def inputs(name):
    return si.make_config(name)


def sample_rows(n, count, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(count, n), replace=False)]))
    return rows.astype(np.int64)


def check_build(sq, R, rows=None):
    w = sq.build_int4(to_dev(R), group=G)
    torch.cuda.synchronize()
    assert w.fmt == sq.SQ_FMT_INT4_G64
    sel = slice(None) if rows is None else rows
    oc, os_, of = oracle.build_int4(R[sel], group=G)
    codes, scales, frac = host(w.codes)[sel], bits16(w.scales)[sel], host(w.frac_idx)[sel]
    assert np.array_equal(codes, oc), first_mismatch(codes, oc)
    assert np.array_equal(scales, os_), first_mismatch(scales, os_)
    assert np.array_equal(frac, of), first_mismatch(frac, of)


@pytest.mark.parametrize("name", ["tiny_64x256x512", "proj_1536x3072x3072", "qkv_1536x9216x3072"])
def test_build_int4_g64(sq, name):
    check_build(sq, inputs(name)["R"])


def test_build_int4_g64_zero_rows_and_unequal_halves(sq):
    """An all-zero row (every group: scale 0, codes 0, fraction 0) and groups whose
    two 32-value halves differ by three orders of magnitude."""
    d = si.make_inputs(4, 768, 384, 31)
    R = d["R"].copy()
    R[3, :] = 0.0
    R[5, 256:512] *= np.float32(1e-3)
    check_build(sq, R)


def check_fwd(sq, d, rows=None, lora=True):
    M, K = d["x"].shape
    N = d["R"].shape[0]
    U = bf16_dev(d["U"]) if lora else None
    D = bf16_dev(d["D"]) if lora else None
    w = sq.build_int4(to_dev(d["R"]), U, D, group=G)
    y = sq.linear_fwd(w, bf16_dev(d["x"]))
    torch.cuda.synchronize()
    rows = np.arange(M, dtype=np.int64) if rows is None else rows
    codes, scales, _ = oracle.build_int4(d["R"], group=G)
    _, _, _, t = oracle.act_quant_nvfp4(d["x"], d["D"])
    xr = oracle.rotate_rows_bf16(d["x"])
    y_ref = oracle.linear_fwd_int4(xr, codes, scales, t if lora else None, d["U"] if lora else None,
                                   M, N, K, rows, group=G)
    y_gpu = host(y)[rows]
    assert np.all(np.isfinite(y_gpu))
    err = norm_err(y_gpu, y_ref)
    assert err <= FWD_TOL, f"normalised error {err:.3e}"


def test_linear_fwd_g64_tiny(sq):
    check_fwd(sq, inputs("tiny_64x256x512"))


def test_linear_fwd_g64_proj_sampled(sq):
    d = inputs("proj_1536x3072x3072")
    check_fwd(sq, d, sample_rows(d["x"].shape[0], 32, 41))


@pytest.mark.parametrize("shape", [(1, 256, 128), (127, 512, 384), (300, 1280, 512)])
def test_linear_fwd_g64_edge_shapes(sq, shape):
    M, K, N = shape
    check_fwd(sq, si.make_inputs(M, K, N, 200 + M))


def test_linear_fwd_g64_ring_slot_reuse(sq):
    """M = 2560 (10 M tiles) and N = 4096 (16 W tiles): the GEMM's W ring has ceil(74 / 10) + 2
    = 10 slots, so six slots take a second W tile.  Sampled rows, the last M tile's among them."""
    d = si.make_inputs(2560, 512, 4096, 244)
    rows = np.unique(np.concatenate([sample_rows(2560, 40, 45), np.arange(2552, 2560)])).astype(np.int64)
    check_fwd(sq, d, rows)


def test_linear_fwd_g64_without_lowrank(sq):
    check_fwd(sq, si.make_inputs(150, 512, 256, 43), lora=False)


def check_reconstruct(sq, d, residual_only=False):
    N, K = d["R"].shape
    w = sq.build_int4(to_dev(d["R"]), bf16_dev(d["U"]), bf16_dev(d["D"]), group=G)
    W = sq.reconstruct_bf16(w, residual_only=residual_only)
    torch.cuda.synchronize()
    c, s, _ = oracle.build_int4(d["R"], group=G)
    Wo = oracle.reconstruct_bf16(oracle.FMT_INT4_G64, c, s, 0.0, d["U"], d["D"], N, K, residual_only)
    Wg = bits16(W)
    assert np.array_equal(Wg, Wo), first_mismatch(Wg, Wo)


@pytest.mark.parametrize("name", ["tiny_64x256x512", "proj_1536x3072x3072"])
def test_reconstruct_g64(sq, name):
    check_reconstruct(sq, inputs(name))


def test_reconstruct_g64_residual_only_ragged(sq):
    check_reconstruct(sq, si.make_inputs(8, 768, 384, 45), residual_only=True)


@pytest.mark.slow
def test_large_g64_sampled(sq):
    """The bench workload 4480 x 16384 x 6144: builder on sampled rows, forward on sampled
    outputs, the whole reconstruct bit for bit."""
    d = inputs("large_4480x16384x6144")
    N = d["R"].shape[0]
    check_build(sq, d["R"], sample_rows(N, 48, 46))
    check_fwd(sq, d, sample_rows(d["x"].shape[0], 6, 47))
    check_reconstruct(sq, d)
