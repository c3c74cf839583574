"""CUDA path vs the CPU oracle on the same seeded inputs, through the C ABI.

Every output of every entry point (sq_build_int4, sq_build_nvfp4,
sq_act_quant_nvfp4, sq_linear_fwd for both codecs, sq_reconstruct_bf16) is
compared with the oracle: integer / packed outputs and the bf16 reconstruct
bit for bit, forward outputs within max|dy| / max|y| <= 2e-3.  Small configs
are compared in full; the full-size configs on sampled rows (rows are
independent everywhere except for the per-tensor global scales, which the
oracle computes over the whole tensor).
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from sqcase import FWD_TOL, bf16_dev, bits16, first_mismatch, host, norm_err, to_dev

pytestmark = pytest.mark.gpu

FULL = ["tiny_64x256x512"]
SAMPLED = ["proj_1536x3072x3072", "qkv_1536x9216x3072"]
LARGE = ["large_4480x6144x6144", "large_4480x16384x6144", "down_4480x6144x16384"]


@pytest.fixture(scope="module")
def sq():
    import bit_quantized_frozen_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


@functools.lru_cache(maxsize=2)
def inputs(name):
    return si.make_config(name)


def sample_rows(n, count, seed):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(count, n), replace=False)]))
    return rows.astype(np.int64)


def sf_matrix(sf_tiled, rows, K):
    C = K // 16
    r = np.asarray(rows, np.int64)[:, None]
    c = np.arange(C, dtype=np.int64)[None, :]
    off = ((r // 128) * (C // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)
    return sf_tiled[off]


# ---------------------------------------------------------------------------
# builders
# ---------------------------------------------------------------------------

def check_int4_build(sq, R, rows=None):
    N, K = R.shape
    w = sq.build_int4(to_dev(R))
    torch.cuda.synchronize()
    codes, scales, frac = host(w.codes), bits16(w.scales), host(w.frac_idx)
    sel = slice(None) if rows is None else rows
    oc, os_, of = oracle.build_int4(R[sel])
    assert np.array_equal(codes[sel], oc), first_mismatch(codes[sel], oc)
    assert np.array_equal(scales[sel], os_), first_mismatch(scales[sel], os_)
    assert np.array_equal(frac[sel], of), first_mismatch(frac[sel], of)


def check_nvfp4_build(sq, R, rows=None):
    N, K = R.shape
    w = sq.build_nvfp4(to_dev(R))
    torch.cuda.synchronize()
    codes, sf, g = host(w.codes), host(w.scales), host(w.g_w)[0]
    if rows is None:
        oc, osf, og = oracle.build_nvfp4(R)
        assert g == og
        assert np.array_equal(codes, oc), first_mismatch(codes, oc)
        assert np.array_equal(sf, osf), first_mismatch(sf, osf)
    else:
        rot = oracle.rotate_rows_f32(R)
        og = oracle.nvfp4_global_scale(np.abs(rot).max())
        assert g == og
        oc, osf = oracle.nvfp4_quant_rotated(rot[rows], og)
        assert np.array_equal(codes[rows], oc), first_mismatch(codes[rows], oc)
        got = sf_matrix(sf, rows, K)
        want = sf_matrix(osf, np.arange(len(rows)), K)
        assert np.array_equal(got, want), first_mismatch(got, want)


@pytest.mark.parametrize("name", FULL + SAMPLED)
def test_build_int4(sq, name):
    check_int4_build(sq, inputs(name)["R"])


@pytest.mark.parametrize("name", FULL + SAMPLED)
def test_build_nvfp4(sq, name):
    check_nvfp4_build(sq, inputs(name)["R"])


# ---------------------------------------------------------------------------
# activation quantisation
# ---------------------------------------------------------------------------

def check_act_quant(sq, x_bits, D_bits, static_g=None):
    M, K = x_bits.shape
    x = bf16_dev(x_bits)
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.full((sq.sq_sf_bytes(M, K),), 0xAB, dtype=torch.uint8, device="cuda")   # poison padding
    g = torch.tensor([0.0 if static_g is None else static_g], dtype=torch.float32, device="cuda")
    t = torch.empty((M, 32), dtype=torch.float32, device="cuda") if D_bits is not None else None
    D = bf16_dev(D_bits) if D_bits is not None else None
    ws = sq.workspace(sq.SQ_OP_ACT_QUANT_NVFP4, M, 0, K)
    sq.sq_act_quant_nvfp4(x, codes, sf, g, D, t, flags=sq.SQ_ACT_STATIC_SCALE if static_g is not None else 0,
                          ws=ws)
    torch.cuda.synchronize()
    oc, osf, og, ot = oracle.act_quant_nvfp4(x_bits, D_bits, static_g)
    assert host(g)[0] == og
    assert np.array_equal(host(codes), oc), first_mismatch(host(codes), oc)
    assert np.array_equal(host(sf), osf), first_mismatch(host(sf), osf)
    if t is not None:
        err = norm_err(host(t), ot)
        assert err < 1e-5, err


@pytest.mark.parametrize("name", FULL + SAMPLED)
def test_act_quant(sq, name):
    d = inputs(name)
    check_act_quant(sq, d["x"], d["D"])


def test_act_quant_static_scale_and_ragged_rows(sq):
    d = si.make_inputs(77, 512, 128, 5)
    check_act_quant(sq, d["x"], None, static_g=0.0017)
    check_act_quant(sq, d["x"], d["D"])


# ---------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------

def gpu_weight(sq, d, fmt, lora=True):
    R = to_dev(d["R"])
    U = bf16_dev(d["U"]) if lora else None
    D = bf16_dev(d["D"]) if lora else None
    if fmt == sq.SQ_FMT_NVFP4:
        return sq.build_nvfp4(R, U, D)
    return sq.build_int4(R, U, D)


def oracle_fwd(d, fmt, rows, lora=True, static_g=None):
    M, K = d["x"].shape
    N = d["R"].shape[0]
    _, _, _, t = oracle.act_quant_nvfp4(d["x"], d["D"])
    t = t if lora else None
    U = d["U"] if lora else None
    if fmt == 2:
        wc, wsf, gw = oracle.build_nvfp4(d["R"])
        xc, xsf, gx, _ = oracle.act_quant_nvfp4(d["x"], None, static_g)
        return oracle.linear_fwd_nvfp4(xc, xsf, gx, wc, wsf, gw, t, U, M, N, K, rows), gx
    codes, scales, _ = oracle.build_int4(d["R"])
    xr = oracle.rotate_rows_bf16(d["x"])
    return oracle.linear_fwd_int4(xr, codes, scales, t, U, M, N, K, rows), None


def check_fwd(sq, d, fmt, rows=None, lora=True, static_g=None):
    M = d["x"].shape[0]
    w = gpu_weight(sq, d, fmt, lora)
    x = bf16_dev(d["x"])
    g_x = torch.tensor([static_g if static_g is not None else 0.0], dtype=torch.float32, device="cuda")
    y = sq.linear_fwd(w, x, g_x=g_x, flags=sq.SQ_ACT_STATIC_SCALE if static_g is not None else 0)
    torch.cuda.synchronize()
    rows = np.arange(M, dtype=np.int64) if rows is None else rows
    y_ref, gx = oracle_fwd(d, fmt, rows, lora, static_g)
    if gx is not None:
        assert host(g_x)[0] == gx
    y_gpu = host(y)[rows]
    assert np.all(np.isfinite(y_gpu))
    err = norm_err(y_gpu, y_ref)
    assert err <= FWD_TOL, f"normalised error {err:.3e}"
    return err


@pytest.mark.parametrize("fmt", [2, 1], ids=["nvfp4", "int4"])
@pytest.mark.parametrize("name", FULL + SAMPLED)
def test_linear_fwd(sq, name, fmt):
    d = inputs(name)
    M = d["x"].shape[0]
    rows = None if name in FULL else sample_rows(M, 48, 7)
    check_fwd(sq, d, fmt, rows)


@pytest.mark.parametrize("fmt", [2, 1], ids=["nvfp4", "int4"])
@pytest.mark.parametrize("shape", [(1, 256, 128), (127, 512, 384), (200, 768, 256), (129, 256, 640),
                                   (300, 1280, 512)])
def test_linear_fwd_edge_shapes(sq, shape, fmt):
    M, K, N = shape
    d = si.make_inputs(M, K, N, 100 + M)
    check_fwd(sq, d, fmt)


@pytest.mark.parametrize("fmt", [2, 1], ids=["nvfp4", "int4"])
def test_linear_fwd_without_lowrank(sq, fmt):
    d = si.make_inputs(150, 512, 256, 11)
    check_fwd(sq, d, fmt, lora=False)


def test_linear_fwd_static_activation_scale(sq):
    d = si.make_inputs(96, 512, 256, 12)
    check_fwd(sq, d, 2, static_g=0.004)


@pytest.mark.parametrize("fmt", [2, 1], ids=["nvfp4", "int4"])
def test_linear_fwd_zero_residual_is_lowrank_only(sq, fmt):
    d = si.make_inputs(64, 512, 256, 13, dist="zero")
    check_fwd(sq, d, fmt)


@pytest.mark.parametrize("fmt", [2, 1, 4], ids=["nvfp4", "int4", "int8"])
@pytest.mark.parametrize("shape", [(300, 1280, 512), (64, 512, 256)])
def test_linear_fwd_bf16_output(sq, shape, fmt):
    """SQ_OUT_BF16: y is the round-to-nearest-even of the fp32 output, bit for bit (one rounding
    of the same value, in the GEMM's epilogue), for every payload format and a ragged M."""
    M, K, N = shape
    d = si.make_inputs(M, K, N, 15 + M)
    if fmt == 4:
        w = sq.build_int8(to_dev(d["R"]), bf16_dev(np.ascontiguousarray(d["U"][:, :16])),
                          bf16_dev(np.ascontiguousarray(d["D"][:, :16])))
    else:
        w = gpu_weight(sq, d, fmt)
    x = bf16_dev(d["x"])
    y32 = sq.linear_fwd(w, x)
    y16 = sq.linear_fwd(w, x, out_bf16=True)
    torch.cuda.synchronize()
    assert y16.dtype == torch.bfloat16 and tuple(y16.shape) == (M, N)
    want = si.to_bf16_bits(host(y32))
    got = bits16(y16)
    assert np.array_equal(got, want), first_mismatch(got, want)


def test_linear_fwd_zero_activation(sq):
    d = si.make_inputs(64, 512, 256, 14)
    d["x"][:] = 0
    w = gpu_weight(sq, d, 2)
    y = sq.linear_fwd(w, bf16_dev(d["x"]))
    torch.cuda.synchronize()
    assert not host(y).any()


# ---------------------------------------------------------------------------
# reconstruct
# ---------------------------------------------------------------------------

def check_reconstruct(sq, d, fmt, residual_only=False, rows=None):
    N, K = d["R"].shape
    w = gpu_weight(sq, d, fmt)
    W = sq.reconstruct_bf16(w, residual_only=residual_only)
    torch.cuda.synchronize()
    sel = slice(None) if rows is None else rows
    if fmt == 2:
        c, s, g = oracle.build_nvfp4(d["R"])
    else:
        c, s, _ = oracle.build_int4(d["R"])
        g = 0.0
    U, Dd = d["U"], d["D"]
    if rows is not None:
        if fmt == 2:
            s = np.concatenate([sf_matrix(s, rows, K)])  # per-row scales, re-tiled below
            s_t = np.zeros(oracle.sf_bytes(len(rows), K), np.uint8)
            C = K // 16
            for i in range(len(rows)):
                for cc in range(C):
                    s_t[oracle.sf_offset(i, cc, C)] = s[i, cc]
            s = s_t
        else:
            s = s[rows]
        c = c[rows]
        U = U[rows]
    Wo = oracle.reconstruct_bf16(fmt, c, s, g, U, Dd, len(c), K, residual_only)
    Wg = bits16(W)[sel]
    assert np.array_equal(Wg, Wo), first_mismatch(Wg, Wo)


@pytest.mark.parametrize("fmt", [2, 1], ids=["nvfp4", "int4"])
@pytest.mark.parametrize("name", FULL + SAMPLED)
def test_reconstruct(sq, name, fmt):
    check_reconstruct(sq, inputs(name), fmt)


@pytest.mark.parametrize("fmt", [2, 1], ids=["nvfp4", "int4"])
def test_reconstruct_residual_only(sq, fmt):
    check_reconstruct(sq, si.make_inputs(8, 768, 384, 15), fmt, residual_only=True)


# ---------------------------------------------------------------------------
# full-size configs: sampled rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", LARGE)
def test_large_builders_sampled(sq, name):
    d = inputs(name)
    N = d["R"].shape[0]
    rows = sample_rows(N, 24, 21)
    check_int4_build(sq, d["R"], rows)
    check_nvfp4_build(sq, d["R"], rows)


def last_tile_rows(M, count, seed):
    """Rows of the last 256-row GEMM tile (the half-empty one when M % 256 == 128)."""
    lo = (M - 1) // 256 * 256
    rng = np.random.default_rng(seed)
    return rng.choice(np.arange(lo, M), size=min(count, M - lo), replace=False)


@pytest.mark.parametrize("fmt", [2, 1], ids=["nvfp4", "int4"])
@pytest.mark.parametrize("name", LARGE)
def test_large_forward_sampled(sq, name, fmt):
    """64 sampled rows of the full-size forward, 8 of them from the last 256-row tile."""
    d = inputs(name)
    M = d["x"].shape[0]
    rows = np.unique(np.concatenate([sample_rows(M, 56, 22), last_tile_rows(M, 8, 25)])).astype(np.int64)
    assert len(rows) >= 64 and rows.max() >= (M - 1) // 256 * 256
    check_fwd(sq, d, fmt, rows)


@pytest.mark.parametrize("name", LARGE)
def test_large_act_quant_bit_exact(sq, name):
    """The activation quantisation at M = 4480 in full: every code, every tiled scale byte
    (padding included) and g_x bit for bit, t within 1e-5 of the fp64 sum."""
    d = inputs(name)
    check_act_quant(sq, d["x"], d["D"])


@pytest.mark.parametrize("M", [9472, 9600], ids=["split-k", "unsplit"])
def test_act_quant_unsplit_first_pass(sq, M):
    """M = 9600 has 75 tiles of 128 rows, more than half the SMs, so the pass that takes the
    absmax and t runs without splitting K (t written in one piece); M = 9472 (74 tiles) still splits
    K in two.  Both bit-exact against the oracle, t within 1e-5."""
    rng = np.random.default_rng(26)
    K = 512
    x = si.to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32) * np.float32(1.5))
    D = si.to_bf16_bits(rng.standard_normal((K, 32), dtype=np.float32) * np.float32(0.02))
    check_act_quant(sq, x, D)


@pytest.mark.parametrize("name", LARGE)
def test_large_reconstruct_sampled(sq, name):
    d = inputs(name)
    N = d["R"].shape[0]
    check_reconstruct(sq, d, 1, rows=sample_rows(N, 12, 23))
    check_reconstruct(sq, d, 2, rows=sample_rows(N, 12, 24))
