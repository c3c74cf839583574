"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every entry point that include/sq.h declares, computes its size helpers, and
rejects bad arguments with the documented status before touching the device.
Fault injection happens on the host only (NULL, misaligned and mis-shaped
arguments, an undersized workspace, a missing device)."""
import ctypes
import os
import re

import pytest
import torch

import bit_quantized_frozen_b200 as sq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sq.h")

SQ_ERR_NULL, SQ_ERR_SHAPE, SQ_ERR_ALIGN, SQ_ERR_WORKSPACE, SQ_ERR_DEVICE, SQ_ERR_ARG = 1, 2, 3, 4, 5, 7

# fake, never dereferenced device addresses: validation fails before any CUDA call
A = 0x7F0000000000
MIS = A + 8


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^SQ_API[^;(]*?\b(sq_\w+)\s*\(", text, re.M)))


def test_header_declares_the_five_operations():
    names = header_functions()
    for op in ["sq_build_int4", "sq_build_nvfp4", "sq_act_quant_nvfp4", "sq_linear_fwd", "sq_reconstruct_bf16"]:
        assert op in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(sq.LIB_PATH)
    for name in header_functions():
        assert hasattr(L, name), name
    assert sorted(sq.EXPORTED) == header_functions()


def test_debug_library_exports_the_same_symbols():
    """libsq_debug.so (built with SQ_DEBUG_CHECKS) exports every declared entry point too and says
    that it is the checked build; the release library says it is not; the index status has a name."""
    from bit_quantized_frozen_b200 import build as b
    dbg = b.build(debug_checks=True)
    D = ctypes.CDLL(dbg)
    for name in header_functions():
        assert hasattr(D, name), name
    D.sq_debug_checks.restype = ctypes.c_int
    assert D.sq_debug_checks() == 1
    assert sq.sq_debug_checks() == 0
    assert sq.status_str(10) == "device index check failed"
    D.sq_selftest_index_check.restype = ctypes.c_int
    assert D.sq_selftest_index_check(None, None) == SQ_ERR_NULL
    assert D.sq_selftest_index_check(ctypes.c_void_p(MIS), None) == SQ_ERR_ALIGN


def test_size_helpers():
    assert sq.sq_abi_version() == 1
    assert sq.sq_sf_bytes(1, 256) == 128 * 16
    assert sq.sq_sf_bytes(128, 512) == 128 * 32
    assert sq.sq_sf_bytes(129, 512) == 256 * 32
    assert sq.sq_sf_bytes(4480, 6144) == 4480 * 384
    assert sq.sq_workspace_bytes(sq.SQ_OP_BUILD_NVFP4, 0, 256, 512) >= 8
    ws = sq.sq_workspace_bytes(sq.SQ_OP_LINEAR_FWD_NVFP4, 64, 256, 512)
    # activation codes + scales, fp32 t, [t_hi | t_lo], [U | U]
    assert ws >= 64 * 256 + sq.sq_sf_bytes(64, 512) + 64 * 32 * 4 + 64 * 128 + 256 * 128
    # int4: bf16(H x), fp32 t, [t_hi | t_lo], [U | U] and the GEMM's ring of dequantised
    # 256-row W tiles (as many as are in flight: 7 at M = 4480); no bf16 copy of W, so
    # doubling N adds only the [U | U] rows
    wsi = sq.sq_workspace_bytes(sq.SQ_OP_LINEAR_FWD_INT4, 64, 256, 512)
    assert wsi >= 64 * 512 * 2 + 64 * 32 * 4 + 64 * 128 + 256 * 128 + 256 * 512 * 2
    for op in (sq.SQ_OP_LINEAR_FWD_INT4, sq.SQ_OP_LINEAR_FWD_INT8):
        grow = sq.sq_workspace_bytes(op, 4480, 4096, 4096) - sq.sq_workspace_bytes(op, 4480, 2048, 4096)
        assert 2048 * 128 <= grow <= 2048 * 128 * 2 + 4096
        ring7 = 7 * 256 * 4096 * 2
        assert sq.sq_workspace_bytes(op, 4480, 4096, 4096) >= 4480 * 4096 * 2 + ring7
    # int8: the int4 layout plus the rank-16 factors widened to rank 32
    assert sq.sq_workspace_bytes(sq.SQ_OP_LINEAR_FWD_INT8, 64, 256, 512) >= wsi + (512 + 256) * 64
    assert sq.sq_workspace_bytes(99, 1, 1, 1) == 0
    assert sq.status_str(0) == "ok"
    assert sq.status_str(2) == "unsupported shape"


def _int4(R=A, N=256, K=512, group=32, codes=A, scales=A, frac=None):
    return sq.lib().sq_build_int4(R, N, K, group, codes, scales, frac, None)


def test_build_int4_validation():
    assert _int4(R=None) == SQ_ERR_NULL
    assert _int4(codes=None) == SQ_ERR_NULL
    assert _int4(K=300) == SQ_ERR_SHAPE
    assert _int4(N=100) == SQ_ERR_SHAPE
    assert _int4(group=16) == SQ_ERR_SHAPE
    assert _int4(group=128) == SQ_ERR_SHAPE
    assert _int4(R=MIS) == SQ_ERR_ALIGN
    assert _int4(frac=MIS) == SQ_ERR_ALIGN


def test_build_int8_validation():
    L = sq.lib()
    assert L.sq_build_int8(None, 256, 512, A, A, None, None) == SQ_ERR_NULL
    assert L.sq_build_int8(A, 256, 512, None, A, None, None) == SQ_ERR_NULL
    assert L.sq_build_int8(A, 256, 300, A, A, None, None) == SQ_ERR_SHAPE
    assert L.sq_build_int8(A, 256, 16384 + 256, A, A, None, None) == SQ_ERR_SHAPE   # one rotated row in smem
    assert L.sq_build_int8(A, 100, 512, A, A, None, None) == SQ_ERR_SHAPE
    assert L.sq_build_int8(MIS, 256, 512, A, A, None, None) == SQ_ERR_ALIGN
    assert L.sq_build_int8(A, 256, 512, A, A + 2, None, None) == SQ_ERR_ALIGN


def test_svd_init_validation():
    L = sq.lib()
    big = 1 << 30
    svd = lambda W=A, N=256, K=512, om=A, it=4, rk=32, ws=A, wsb=big: \
        L.sq_svd_init(W, N, K, om, it, rk, A, A, A, ws, wsb, None)
    assert svd(W=None) == SQ_ERR_NULL
    assert svd(K=300) == SQ_ERR_SHAPE
    assert svd(it=0) == SQ_ERR_ARG
    assert svd(it=101) == SQ_ERR_ARG
    assert svd(rk=8) == SQ_ERR_ARG
    assert svd(rk=24) == SQ_ERR_ARG
    assert svd(om=MIS) == SQ_ERR_ALIGN
    assert svd(wsb=64) == SQ_ERR_WORKSPACE
    assert sq.sq_workspace_bytes(sq.SQ_OP_SVD_INIT, 0, 256, 512) >= (256 + 512) * 32 * 4


def test_build_nvfp4_validation():
    L = sq.lib()
    assert L.sq_build_nvfp4(A, 256, 512, A, A, A, None, 256, None) == SQ_ERR_NULL
    assert L.sq_build_nvfp4(A, 256, 250, A, A, A, A, 256, None) == SQ_ERR_SHAPE
    assert L.sq_build_nvfp4(A, 256, 512, A, A, A, A + 16, 256, None) == SQ_ERR_ALIGN
    assert L.sq_build_nvfp4(A, 256, 512, A, A, A, A, 4, None) == SQ_ERR_WORKSPACE


def test_act_quant_validation():
    L = sq.lib()
    big = 1 << 30
    assert L.sq_act_quant_nvfp4(None, 4, 512, A, A, A, None, None, 0, A, big, None) == SQ_ERR_NULL
    assert L.sq_act_quant_nvfp4(A, 0, 512, A, A, A, None, None, 0, A, big, None) == SQ_ERR_SHAPE
    assert L.sq_act_quant_nvfp4(A, 4, 512, A, A, A, None, None, 0x80, A, big, None) == SQ_ERR_ARG
    assert L.sq_act_quant_nvfp4(A, 4, 512, A, A, A, None, MIS, 0, A, big, None) == SQ_ERR_ALIGN
    assert L.sq_act_quant_nvfp4(A, 4, 512, A, A, A, None, None, 0, A, 16, None) == SQ_ERR_WORKSPACE


def _w(fmt=sq.SQ_FMT_NVFP4, N=256, K=512, codes=A, scales=A, g_w=A, U=A, D=A):
    return sq.sq_weight(fmt, N, K, codes, scales, g_w, U, D)


def test_linear_fwd_validation():
    L = sq.lib()
    big = 1 << 34
    fwd = lambda w, x=A, M=8, y=A, gx=None, fl=0, ws=A, wsb=big: L.sq_linear_fwd(
        ctypes.byref(w), x, M, y, gx, fl, ws, wsb, None)
    assert fwd(_w(codes=None)) == SQ_ERR_NULL
    assert fwd(_w(g_w=None)) == SQ_ERR_NULL
    assert fwd(_w(fmt=7)) == SQ_ERR_ARG
    assert fwd(_w(fmt=sq.SQ_FMT_INT8_ROW, K=16384 + 256, g_w=None)) == SQ_ERR_SHAPE
    assert fwd(_w(N=192)) == SQ_ERR_SHAPE
    assert fwd(_w(), M=0) == SQ_ERR_SHAPE
    assert fwd(_w(), y=MIS) == SQ_ERR_ALIGN
    assert fwd(_w(), ws=A + 64) == SQ_ERR_ALIGN
    assert fwd(_w(), wsb=100) == SQ_ERR_WORKSPACE
    assert fwd(_w(), fl=sq.SQ_ACT_STATIC_SCALE) == SQ_ERR_NULL          # static scale needs g_x
    assert fwd(_w(), fl=0x20) == SQ_ERR_ARG                             # unknown flag
    assert fwd(_w(fmt=sq.SQ_FMT_INT4_G32, g_w=None), gx=A, fl=sq.SQ_ACT_STATIC_SCALE) == SQ_ERR_ARG
    assert fwd(_w(), fl=0x40) == SQ_ERR_ARG


def test_bwd_dx_validation():
    L = sq.lib()
    big = 1 << 34
    bwd = lambda w, dy=A, M=8, dx=A, ws=A, wsb=big: L.sq_linear_bwd_dx(ctypes.byref(w), dy, M, dx, ws, wsb, None)
    assert bwd(_w(), dy=None) == SQ_ERR_NULL
    assert bwd(_w(), M=0) == SQ_ERR_SHAPE
    assert bwd(_w(N=200)) == SQ_ERR_SHAPE
    assert bwd(_w(), dx=MIS) == SQ_ERR_ALIGN
    assert bwd(_w(), wsb=1000) == SQ_ERR_WORKSPACE
    assert sq.sq_workspace_bytes(sq.SQ_OP_LINEAR_BWD_DX, 8, 256, 512) >= 256 * 512 * 2


def test_reconstruct_validation():
    L = sq.lib()
    assert L.sq_reconstruct_bf16(ctypes.byref(_w()), None, 0, None) == SQ_ERR_NULL
    assert L.sq_reconstruct_bf16(ctypes.byref(_w()), MIS, 0, None) == SQ_ERR_ALIGN
    assert L.sq_reconstruct_bf16(ctypes.byref(_w()), A, 0x10, None) == SQ_ERR_ARG
    assert L.sq_reconstruct_bf16(ctypes.byref(_w()), A, 0x8, None) == SQ_ERR_ARG
    assert L.sq_reconstruct_bf16(ctypes.byref(_w(U=MIS)), A, 0, None) == SQ_ERR_ALIGN


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_device_error():
    assert _int4() == SQ_ERR_DEVICE
    assert _int4(group=64) == SQ_ERR_DEVICE            # group 64 passes validation
    assert sq.lib().sq_build_int8(A, 256, 512, A, A, None, None) == SQ_ERR_DEVICE
    assert sq.lib().sq_reconstruct_bf16(ctypes.byref(_w(fmt=sq.SQ_FMT_INT8_ROW, g_w=None)), A, 0, None) \
        == SQ_ERR_DEVICE
    assert sq.lib().sq_reconstruct_bf16(ctypes.byref(_w(fmt=sq.SQ_FMT_INT4_G64, g_w=None)), A, 0, None) \
        == SQ_ERR_DEVICE
    assert sq.lib().sq_reconstruct_bf16(ctypes.byref(_w()), A, 0, None) == SQ_ERR_DEVICE
    # the library's own status word (ws == NULL) needs a device too
    assert sq.lib().sq_check_device_status(None, None) == SQ_ERR_DEVICE
    assert sq.lib().sq_check_device_status(MIS, None) == SQ_ERR_ALIGN


def test_selftest_validation():
    L = sq.lib()
    assert L.sq_selftest_wait_timeout(None, 100, None) == SQ_ERR_NULL
    assert L.sq_selftest_wait_timeout(MIS, 100, None) == SQ_ERR_ALIGN
    assert L.sq_selftest_wait_timeout(A, 0, None) == SQ_ERR_ARG
    assert L.sq_selftest_wait_timeout(A, 2000000, None) == SQ_ERR_ARG


def test_binding_raises_with_status():
    with pytest.raises(sq.SqError) as e:
        sq._check("sq_build_int4", SQ_ERR_SHAPE)
    assert e.value.status == SQ_ERR_SHAPE


def test_nonfinite_guard_flag_and_status():
    L = sq.lib()
    assert L.sq_status_str(9) == b"non-finite input"
    big = 1 << 34
    # the flag passes validation (no device here: the device check answers)
    fl = sq.SQ_CHECK_FINITE | sq.SQ_OUT_BF16
    want = SQ_ERR_DEVICE if not torch.cuda.is_available() else None
    if want is not None:
        assert L.sq_linear_fwd(ctypes.byref(_w()), A, 8, A, None, fl, A, big, None) == want
        assert L.sq_act_quant_nvfp4(A, 4, 512, A, A, A, None, None, sq.SQ_CHECK_FINITE, A, big, None) == want



C_PROGRAM = r"""
#include "sq.h"
#include <stdio.h>
#include <string.h>

/* every entry point, by address: the header is plain C and the library exports them all */
typedef void (*fnptr)(void);
static const fnptr entries[] = {
    (fnptr)sq_status_str, (fnptr)sq_abi_version, (fnptr)sq_last_error_detail, (fnptr)sq_sf_bytes,
    (fnptr)sq_workspace_bytes, (fnptr)sq_build_int4, (fnptr)sq_svd_init, (fnptr)sq_build_int8,
    (fnptr)sq_build_nvfp4, (fnptr)sq_act_quant_nvfp4, (fnptr)sq_linear_fwd, (fnptr)sq_linear_fwd_noalloc,
    (fnptr)sq_reconstruct_bf16, (fnptr)sq_linear_bwd_dx, (fnptr)sq_set_gemm_events, (fnptr)sq_set_stage_events,
    (fnptr)sq_check_device_status, (fnptr)sq_selftest_wait_timeout, (fnptr)sq_debug_checks,
    (fnptr)sq_selftest_index_check,
};

int main(void)
{
    sq_weight w;
    size_t i;
    for (i = 0; i < sizeof(entries) / sizeof(entries[0]); ++i)
        if (!entries[i])
            return 1;
    memset(&w, 0, sizeof(w));
    w.fmt = SQ_FMT_NVFP4;
    w.N = 256;
    w.K = 512;
    /* host-side validation only: no device is touched */
    if (sq_linear_fwd(&w, NULL, 8, NULL, NULL, 0, NULL, 0, NULL) != SQ_ERR_NULL)
        return 2;
    if (sq_build_int4(NULL, 256, 512, 32, NULL, NULL, NULL, NULL) != SQ_ERR_NULL)
        return 3;
    if (sq_sf_bytes(130, 512) != 256 * 32)
        return 4;
    printf("%d %s\n", sq_abi_version(), sq_status_str(SQ_ERR_NONFINITE));
    return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    """include/sq.h compiles as strict C99 (-pedantic, warnings as errors), a C program links
    against libsq.so, takes the address of every entry point and runs the host-side checks."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_sq.c"
    exe = tmp_path / "use_sq"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(sq.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                    os.path.join(ROOT, "include"), str(src), "-L", libdir, "-lsq", "-Wl,-rpath," + libdir,
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    assert out.split() == ["1", "non-finite", "input"]
    text = open(HEADER).read()
    assert len(header_functions()) == C_PROGRAM.count("(fnptr)sq_")
    assert "namespace" not in text and "torch" not in text
