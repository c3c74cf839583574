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

SCRATCH_BYTES = 96 << 20


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
                                      ("tiny_64x256x512", 1), ("large_4480x16384x6144", 1)],
                         ids=["proj-nvfp4", "tiny-nvfp4", "tiny-int4", "large-int4"])
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


VARIANTS = {
    # id: (format, flag name or None, pass g_x)
    "nvfp4-no-gx": (2, None, False),
    "nvfp4-bf16-out": (2, "SQ_OUT_BF16", True),
    "nvfp4-static-scale": (2, "SQ_ACT_STATIC_SCALE", True),
    "int4-g64": (3, None, False),
    "int8-row": (4, None, False),
}


@pytest.mark.gpu
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_noalloc_variants_match_workspace_forward(sq, variant):
    """The other layouts the static scratch is carved into: the NVFP4 forward without a g_x
    pointer (the scale then lives inside the scratch), with bf16 output, with a static activation
    scale; the group-64 int4 and the int8 per-row formats (the latter with its widened rank-16
    factors).  Each against sq_linear_fwd with a caller workspace on the same inputs, two calls in
    a row, bit for bit (the same kernels run on the same values), and the scratch's status word
    read back clean."""
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fmt, flag, pass_g = VARIANTS[variant]
    flags = getattr(sq, flag) if flag else 0
    d = si.make_config("tiny_64x256x512")
    M, K = d["x"].shape
    N = d["R"].shape[0]
    R, U, D = to_dev(d["R"]), bf16_dev(d["U"]), bf16_dev(d["D"])
    if fmt == 2:
        w = sq.build_nvfp4(R, U, D)
    elif fmt == 3:
        w = sq.build_int4(R, U, D, group=64)
    else:
        w = sq.build_int8(R, U[:, :16].contiguous(), D[:, :16].contiguous())
    x = bf16_dev(d["x"])
    ydt = torch.bfloat16 if flags & sq.SQ_OUT_BF16 else torch.float32
    static = torch.tensor([0.0123], dtype=torch.float32, device="cuda")

    def g_in():
        if flags & sq.SQ_ACT_STATIC_SCALE:
            return static.clone()
        return torch.full((1,), -1.0, dtype=torch.float32, device="cuda") if pass_g else None

    y_ref = torch.empty((M, N), dtype=ydt, device="cuda")
    op = {2: sq.SQ_OP_LINEAR_FWD_NVFP4, 4: sq.SQ_OP_LINEAR_FWD_INT8}.get(fmt, sq.SQ_OP_LINEAR_FWD_INT4)
    g_ref = g_in()
    sq.sq_linear_fwd(w, x, y_ref, g_x=g_ref, flags=flags, ws=sq.workspace(op, M, N, K))
    torch.cuda.synchronize()
    ref = y_ref.view(torch.int16 if ydt == torch.bfloat16 else torch.int32).cpu().numpy()
    assert np.all(np.isfinite(y_ref.float().cpu().numpy())) and y_ref.float().abs().max().item() > 0
    scratch = []
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=ydt, device="cuda")
        g = g_in()
        scratch.append(sq.sq_linear_fwd_noalloc(w, x, y, g_x=g, flags=flags))
        torch.cuda.synchronize()
        got = y.view(torch.int16 if ydt == torch.bfloat16 else torch.int32).cpu().numpy()
        assert np.array_equal(got, ref), f"{variant}, call {call}: output differs from the workspace forward"
        if g is not None:
            assert host(g)[0] == host(g_ref)[0], f"{variant}, call {call}: g_x differs"
        sq.sq_check_device_status(scratch[-1])
    assert scratch[0] and scratch[0] == scratch[1]


def test_noalloc_rejects_shape_beyond_scratch(sq):
    # int4 at N = 16384, K = 6144 fits M = 6536 rows, not 6537 (NVFP4: 26544, not
    # 26545): refused before any device work (the weight pointers are never touched).
    import ctypes
    fake = 1 << 20
    for fmt, op, m_max in ((sq.SQ_FMT_INT4_G32, sq.SQ_OP_LINEAR_FWD_INT4, 6536),
                           (sq.SQ_FMT_NVFP4, sq.SQ_OP_LINEAR_FWD_NVFP4, 26544)):
        w = sq.sq_weight(fmt, 16384, 6144, fake, fake, fake, fake, fake)
        assert sq.sq_workspace_bytes(op, m_max + 1, 16384, 6144) > SCRATCH_BYTES
        assert sq.sq_workspace_bytes(op, m_max, 16384, 6144) <= SCRATCH_BYTES
        out = ctypes.c_void_p(123)
        st = sq.lib().sq_linear_fwd_noalloc(ctypes.byref(w), fake, m_max + 1, fake, None, 0, ctypes.byref(out), None)
        assert sq.status_str(st) == "workspace too small"
        assert out.value is None
        detail = sq.lib().sq_last_error_detail().decode()
        assert "100663296" in detail and f"M={m_max + 1}" in detail
