"""Every output byte is written, and every op is deterministic.

Each op of the C ABI runs twice on the same inputs, once into outputs filled with 0xFF bytes
and once into outputs filled with 0x5A bytes; the two results must be identical byte for byte
(a byte the kernels leave unwritten keeps its fill and differs).  Identical bytes also show that
the builders, the forward, the reconstruct, the backward and the SVD init give the same result
on every run, whatever the CTA schedule: a restarted build reproduces its output exactly.  The
shapes have a ragged M (not a multiple of the 128-row tiles) and several Hadamard blocks.
"""
import numpy as np
import pytest
import torch

import synth_inputs as si
from sqcase import bf16_dev, to_dev

pytestmark = pytest.mark.gpu

POISONS = (0xFF, 0x5A)
M, K, N = 300, 768, 384


@pytest.fixture(scope="module")
def sq():
    import bit_quantized_frozen_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


@pytest.fixture(scope="module")
def data():
    return si.make_inputs(M, K, N, 90)


def poisoned(shape, dtype, fill):
    t = torch.empty(shape, dtype=dtype, device="cuda")
    t.view(torch.uint8).fill_(fill)
    return t


def same_bytes(outs_a, outs_b):
    torch.cuda.synchronize()
    for a, b in zip(outs_a, outs_b):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def twice(make):
    """make(fill) -> tuple of output tensors; run with both fills and compare byte for byte."""
    a = make(POISONS[0])
    b = make(POISONS[1])
    same_bytes(a, b)
    return a


@pytest.mark.parametrize("group", [32, 64])
def test_build_int4_writes_every_byte(sq, data, group):
    R = to_dev(data["R"])

    def make(f):
        c = poisoned((N, K // 2), torch.uint8, f)
        s = poisoned((N, K // group), torch.float16, f)
        fr = poisoned((N, K // group), torch.uint8, f)
        sq.sq_build_int4(R, c, s, fr, group=group)
        return c, s, fr
    twice(make)


def test_build_nvfp4_writes_every_byte(sq, data):
    R = to_dev(data["R"])
    ws = sq.workspace(sq.SQ_OP_BUILD_NVFP4, 0, N, K)

    def make(f):
        c = poisoned((N, K // 2), torch.uint8, f)
        sf = poisoned((sq.sq_sf_bytes(N, K),), torch.uint8, f)
        g = poisoned((1,), torch.float32, f)
        sq.sq_build_nvfp4(R, c, sf, g, ws)
        return c, sf, g
    twice(make)


def test_build_int8_writes_every_byte(sq, data):
    R = to_dev(data["R"])

    def make(f):
        c = poisoned((N, K), torch.int8, f)
        s = poisoned((N,), torch.float32, f)
        fr = poisoned((N,), torch.uint8, f)
        sq.sq_build_int8(R, c, s, fr)
        return c, s, fr
    twice(make)


def test_act_quant_writes_every_byte(sq, data):
    x, D = bf16_dev(data["x"]), bf16_dev(data["D"])
    ws = sq.workspace(sq.SQ_OP_ACT_QUANT_NVFP4, M, 0, K)

    def make(f):
        c = poisoned((M, K // 2), torch.uint8, f)
        sf = poisoned((sq.sq_sf_bytes(M, K),), torch.uint8, f)     # includes the padding rows
        g = poisoned((1,), torch.float32, f)
        t = poisoned((M, 32), torch.float32, f)
        sq.sq_act_quant_nvfp4(x, c, sf, g, D, t, ws=ws)
        return c, sf, g, t
    twice(make)


def weights(sq, data):
    R, U, D = to_dev(data["R"]), bf16_dev(data["U"]), bf16_dev(data["D"])
    U16, D16 = U[:, :16].contiguous(), D[:, :16].contiguous()
    return {
        "nvfp4": sq.build_nvfp4(R, U, D),
        "int4": sq.build_int4(R, U, D),
        "int4_g64": sq.build_int4(R, U, D, group=64),
        "int8": sq.build_int8(R, U16, D16),
    }


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "int4_g64", "int8"])
@pytest.mark.parametrize("bf16_out", [False, True], ids=["fp32", "bf16"])
def test_forward_writes_every_byte(sq, data, fmt, bf16_out):
    w = weights(sq, data)[fmt]
    x = bf16_dev(data["x"])
    op = {"nvfp4": sq.SQ_OP_LINEAR_FWD_NVFP4, "int8": sq.SQ_OP_LINEAR_FWD_INT8}.get(fmt, sq.SQ_OP_LINEAR_FWD_INT4)
    ws = sq.workspace(op, M, N, K)
    flags = sq.SQ_OUT_BF16 if bf16_out else 0

    def make(f):
        y = poisoned((M, N), torch.bfloat16 if bf16_out else torch.float32, f)
        ws.fill_(f)                                      # stale workspace contents must not matter
        sq.sq_linear_fwd(w, x, y, flags=flags, ws=ws)
        return (y,)
    twice(make)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "int4_g64", "int8"])
@pytest.mark.parametrize("flags", [0, 2, 4, 6], ids=["W", "residual", "Wt", "residual_Wt"])
def test_reconstruct_writes_every_byte(sq, data, fmt, flags):
    w = weights(sq, data)[fmt]
    shape = (K, N) if flags & sq.SQ_RECON_TRANSPOSED else (N, K)

    def make(f):
        W = poisoned(shape, torch.bfloat16, f)
        sq.sq_reconstruct_bf16(w, W, flags)
        return (W,)
    twice(make)


def test_backward_writes_every_byte(sq, data):
    w = weights(sq, data)["nvfp4"]
    dy = bf16_dev(si.to_bf16_bits(np.random.default_rng(91).standard_normal((M, N)).astype(np.float32)))
    ws = sq.workspace(sq.SQ_OP_LINEAR_BWD_DX, M, N, K)

    def make(f):
        dx = poisoned((M, K), torch.float32, f)
        ws.fill_(f)
        sq.sq_linear_bwd_dx(w, dy, dx, ws)
        return (dx,)
    twice(make)


@pytest.mark.parametrize("rank", [32, 16])
def test_svd_init_writes_every_byte(sq, data, rank):
    W = to_dev(data["R"]) + 0.0
    om = to_dev(np.random.default_rng(92).standard_normal((K, 32)).astype(np.float32))
    ws = sq.workspace(sq.SQ_OP_SVD_INIT, 0, N, K)

    def make(f):
        up = poisoned((N, rank), torch.bfloat16, f)
        down = poisoned((K, rank), torch.bfloat16, f)
        R = poisoned((N, K), torch.float32, f)
        ws.fill_(f)
        sq.sq_svd_init(W, om, 4, up, down, R, ws)
        return up, down, R
    twice(make)
