"""sq_linear_fwd_noalloc: the forward on libsq's static per-device scratch.

Called through the C ABI binding and compared with sq_linear_fwd (the same
layer, a caller workspace) on the same inputs, on two calls in a row, within
the forward tolerance.  The file name sorts last so that the check also runs
after every other test has used the library on this device.
"""
import numpy as np
import pytest
import torch

import synth_inputs as si
from sqcase import FWD_TOL, bf16_dev, host, norm_err, to_dev

SCRATCH_BYTES = 32 << 20


@pytest.fixture(scope="module")
def sq():
    import bit_quantized_frozen_b200 as m
    m.lib()
    return m


def _weight(sq, d, fmt):
    R, U, D = to_dev(d["R"]), bf16_dev(d["U"]), bf16_dev(d["D"])
    return sq.build_nvfp4(R, U, D) if fmt == sq.SQ_FMT_NVFP4 else sq.build_int4(R, U, D)


@pytest.mark.gpu
@pytest.mark.parametrize("name,fmt", [("proj_1536x3072x3072", 2), ("tiny_64x256x512", 2),
                                      ("tiny_64x256x512", 1)], ids=["proj-nvfp4", "tiny-nvfp4", "tiny-int4"])
def test_noalloc_matches_workspace_forward(sq, name, fmt):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    d = si.make_config(name)
    M, K = d["x"].shape
    N = d["R"].shape[0]
    op = sq.SQ_OP_LINEAR_FWD_NVFP4 if fmt == 2 else sq.SQ_OP_LINEAR_FWD_INT4
    assert sq.sq_workspace_bytes(op, M, N, K) <= SCRATCH_BYTES
    w = _weight(sq, d, fmt)
    x = bf16_dev(d["x"])

    g_ref = torch.zeros(1, dtype=torch.float32, device="cuda")
    y_ref = sq.linear_fwd(w, x, g_x=g_ref)
    torch.cuda.synchronize()
    yr = host(y_ref)
    assert np.all(np.isfinite(yr)) and np.abs(yr).max() > 0

    scratch = []
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        g = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        scratch.append(sq.sq_linear_fwd_noalloc(w, x, y, g_x=g))
        torch.cuda.synchronize()
        yg = host(y)
        assert np.all(np.isfinite(yg)), f"call {call}: non-finite output"
        err = norm_err(yg, yr.astype(np.float64))
        assert err <= FWD_TOL, f"call {call}: normalised difference {err:.3e}"
        if fmt == 2:
            assert host(g)[0] == host(g_ref)[0], f"call {call}: g_x differs"
    assert scratch[0] and scratch[0] == scratch[1]
    assert scratch[0] % 256 == 0
    sq.sq_check_device_status(scratch[1])


def test_noalloc_rejects_shape_beyond_scratch(sq):
    # NVFP4 at N = 16384, K = 6144 fits M = 8462 rows, not 8463: refused before
    # any device work (the weight pointers are never touched).
    fake = 1 << 20
    w = sq.sq_weight(sq.SQ_FMT_NVFP4, 16384, 6144, fake, fake, fake, fake, fake)
    assert sq.sq_workspace_bytes(sq.SQ_OP_LINEAR_FWD_NVFP4, 8463, 16384, 6144) > SCRATCH_BYTES
    assert sq.sq_workspace_bytes(sq.SQ_OP_LINEAR_FWD_NVFP4, 8462, 16384, 6144) <= SCRATCH_BYTES
    import ctypes
    out = ctypes.c_void_p(123)
    st = sq.lib().sq_linear_fwd_noalloc(ctypes.byref(w), fake, 8463, fake, None, 0, ctypes.byref(out), None)
    assert sq.status_str(st) == "workspace too small"
    assert out.value is None
    detail = sq.lib().sq_last_error_detail().decode()
    assert "33554432" in detail and "M=8463" in detail
