"""CPU oracle for the SquareQ W4 linear layer -- TEST INFRASTRUCTURE ONLY.

Plain scalar C (``sq_oracle.c``, built with ``-O2 -ffp-contract=off`` and no
fast-math) behind a ctypes wrapper that takes and returns numpy arrays.  Only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
use it; the product path (``bit_quantized_frozen_b200``) never imports it and
shares no code with it.

Every routine follows the SquareQ README, section "SquareQ v3 -- W4
(Hadamard-256 + low-rank + int4 / NVFP4)"; the C source states, routine by
routine, which paragraph it follows and the reading taken where the page is
silent.  Parity status: every routine here is pinned by the ``-m "not gpu"``
tests in ``tests/test_oracle_pins*.py`` (closed forms, invariants, library
conversions, brute force); none is "parity unpinned".  ``tests/test_oracle_mutants.py``
plants single mistakes in a scratch copy of this package and checks that a pin
fails for each.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile sq_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
               "-shared", "-Wall", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SIGS = {
    "or_num_threads": ([], ctypes.c_int),
    "or_f32_to_bf16": ([_F], ctypes.c_uint16),
    "or_bf16_to_f32": ([ctypes.c_uint16], _F),
    "or_f32_to_f16": ([_F], ctypes.c_uint16),
    "or_f16_to_f32": ([ctypes.c_uint16], _F),
    "or_f32_to_ue4m3": ([_F], ctypes.c_uint8),
    "or_ue4m3_to_f32": ([ctypes.c_uint8], _F),
    "or_f32_to_e2m1": ([_F], ctypes.c_uint8),
    "or_e2m1_to_f32": ([ctypes.c_uint8], _F),
    "or_fwht256": ([_P], None),
    "or_rotate_rows_f32": ([_P, _I64, _I64, _P], None),
    "or_rotate_rows_bf16": ([_P, _I64, _I64, _P], None),
    "or_int4_fraction": ([ctypes.c_int], _F),
    "or_int4_group32": ([_P, _P, _P, _P], None),
    "or_build_int4": ([_P, _I64, _I64, _P, _P, _P], None),
    "or_int4_group64": ([_P, _P, _P, _P], None),
    "or_build_int4_g": ([_P, _I64, _I64, ctypes.c_int, _P, _P, _P], None),
    "or_linear_fwd_int4_g": ([_P, _P, _P, ctypes.c_int, _P, _P, _I64, _I64, _I64, _P, _I64, _P], None),
    "or_sf_offset": ([_I64, _I64, _I64], _I64),
    "or_sf_bytes": ([_I64, _I64], _I64),
    "or_nvfp4_global_scale": ([_F], _F),
    "or_nvfp4_block16": ([_P, _F, _P, _P], None),
    "or_nvfp4_quant_rotated": ([_P, _I64, _I64, _F, _P, _P], None),
    "or_build_nvfp4": ([_P, _I64, _I64, _P, _P, _P, _P], None),
    "or_act_quant_nvfp4": ([_P, _I64, _I64, ctypes.c_int, _P, _P, _P, _P, _P, _P], None),
    "or_linear_fwd_nvfp4": ([_P, _P, _F, _P, _P, _F, _P, _P, _I64, _I64, _I64, _P, _I64, _P], None),
    "or_linear_fwd_int4": ([_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P], None),
    "or_reconstruct_bf16": ([ctypes.c_int, _P, _P, _F, _P, _P, _I64, _I64, ctypes.c_int, _P], None),
    "or_int8_row": ([_P, _I64, _P, _P, _P], None),
    "or_build_int8": ([_P, _I64, _I64, _P, _P, _P], None),
    "or_linear_fwd_int8": ([_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P], None),
    "or_lowrank_input": ([_P, _I64, _I64, _P, ctypes.c_int, _P], None),
    "or_linear_bwd_dx": ([_P, _P, _I64, _I64, _I64, _P, _I64, _P], None),
    "or_svd_residual": ([_P, _P, _P, _I64, _I64, ctypes.c_int, _P], None),
    "or_f32_to_bf16_n": ([_P, _I64, _P], None),
    "or_f64_to_bf16": ([ctypes.c_double], ctypes.c_uint16),
    "or_svd_top": ([_P, _I64, _I64, ctypes.c_int, ctypes.c_int, _P, _P, _P], ctypes.c_int),
    "or_svd_init": ([_P, _I64, _I64, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P], ctypes.c_int),
}


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        for name, (args, res) in _SIGS.items():
            fn = getattr(_lib, name)
            fn.argtypes = args
            fn.restype = res
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _rows(rows, M):
    """The evaluated rows as int64, all of them if None; each must index one of the M rows."""
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(rows, np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= M):
        raise IndexError(f"rows must lie in [0, {M})")
    return rows


def num_threads() -> int:
    return lib().or_num_threads()


# ---- scalar conversions ---------------------------------------------------

def f32_to_bf16(v) -> int:
    return lib().or_f32_to_bf16(float(np.float32(v)))


def bf16_to_f32(b) -> float:
    return lib().or_bf16_to_f32(int(b))


def f32_to_f16(v) -> int:
    return lib().or_f32_to_f16(float(np.float32(v)))


def f16_to_f32(h) -> float:
    return lib().or_f16_to_f32(int(h))


def f32_to_ue4m3(v) -> int:
    return lib().or_f32_to_ue4m3(float(np.float32(v)))


def ue4m3_to_f32(c) -> float:
    return lib().or_ue4m3_to_f32(int(c))


def f32_to_e2m1(v) -> int:
    return lib().or_f32_to_e2m1(float(np.float32(v)))


def e2m1_to_f32(c) -> float:
    return lib().or_e2m1_to_f32(int(c))


# ---- O1/O2 rotation -------------------------------------------------------

def fwht256(v) -> np.ndarray:
    a = _c(v, np.float32).copy()
    assert a.shape == (256,)
    lib().or_fwht256(_p(a))
    return a


def rotate_rows_f32(R) -> np.ndarray:
    R = _c(R, np.float32)
    rows, K = R.shape
    out = np.empty_like(R)
    lib().or_rotate_rows_f32(_p(R), rows, K, _p(out))
    return out


def rotate_rows_bf16(x_bits) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    rows, K = x.shape
    out = np.empty((rows, K), np.float32)
    lib().or_rotate_rows_bf16(_p(x), rows, K, _p(out))
    return out


# ---- O3 int4 --------------------------------------------------------------

def int4_fraction(j: int) -> float:
    return lib().or_int4_fraction(int(j))


def int4_group32(r):
    r = _c(r, np.float32)
    assert r.shape == (32,)
    q = np.empty(32, np.int8)
    s = np.empty(1, np.uint16)
    j = np.empty(1, np.uint8)
    lib().or_int4_group32(_p(r), _p(q), _p(s), _p(j))
    return q, int(s[0]), int(j[0])


def int4_group64(r):
    r = _c(r, np.float32)
    assert r.shape == (64,)
    q = np.empty(64, np.int8)
    s = np.empty(1, np.uint16)
    j = np.empty(1, np.uint8)
    lib().or_int4_group64(_p(r), _p(q), _p(s), _p(j))
    return q, int(s[0]), int(j[0])


def build_int4(R, group=32):
    """R [N, K] fp32 -> (codes [N, K/2] u8, scales [N, K/group] fp16 bits u16, frac [N, K/group] u8),
    group 32 or 64."""
    R = _c(R, np.float32)
    N, K = R.shape
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // group), np.uint16)
    frac = np.empty((N, K // group), np.uint8)
    if group == 32:
        lib().or_build_int4(_p(R), N, K, _p(codes), _p(scales), _p(frac))
    else:
        lib().or_build_int4_g(_p(R), N, K, int(group), _p(codes), _p(scales), _p(frac))
    return codes, scales, frac


# ---- O4/O5 NVFP4 ----------------------------------------------------------

def sf_offset(r: int, c: int, C: int) -> int:
    return lib().or_sf_offset(r, c, C)


def sf_bytes(rows: int, K: int) -> int:
    return lib().or_sf_bytes(rows, K)


def nvfp4_global_scale(A) -> float:
    return lib().or_nvfp4_global_scale(float(np.float32(A)))


def nvfp4_block16(r, g):
    r = _c(r, np.float32)
    assert r.shape == (16,)
    codes = np.empty(8, np.uint8)
    sf = np.empty(1, np.uint8)
    lib().or_nvfp4_block16(_p(r), float(np.float32(g)), _p(codes), _p(sf))
    return codes, int(sf[0])


def nvfp4_quant_rotated(rot, g):
    rot = _c(rot, np.float32)
    rows, K = rot.shape
    codes = np.empty((rows, K // 2), np.uint8)
    sf = np.empty(sf_bytes(rows, K), np.uint8)
    lib().or_nvfp4_quant_rotated(_p(rot), rows, K, float(np.float32(g)), _p(codes), _p(sf))
    return codes, sf


def build_nvfp4(R):
    """R [N, K] fp32 -> (codes [N, K/2] u8, sf tiled u8, g_w float32)."""
    R = _c(R, np.float32)
    N, K = R.shape
    scratch = np.empty_like(R)
    codes = np.empty((N, K // 2), np.uint8)
    sf = np.empty(sf_bytes(N, K), np.uint8)
    g = np.empty(1, np.float32)
    lib().or_build_nvfp4(_p(R), N, K, _p(scratch), _p(codes), _p(sf), _p(g))
    return codes, sf, np.float32(g[0])


def act_quant_nvfp4(x_bits, lora_down_bits=None, static_g=None):
    """x [M, K] bf16 bits -> (codes, sf tiled, g_x float32, t [M, 32] fp64 or None)."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    scratch = np.empty((M, K), np.float32)
    codes = np.empty((M, K // 2), np.uint8)
    sf = np.empty(sf_bytes(M, K), np.uint8)
    g = np.array([0.0 if static_g is None else static_g], np.float32)
    t = None
    D = None
    if lora_down_bits is not None:
        D = _c(lora_down_bits, np.uint16)
        assert D.shape == (K, 32)
        t = np.empty((M, 32), np.float64)
    lib().or_act_quant_nvfp4(_p(x), M, K, 0 if static_g is None else 1, _p(g), _p(scratch),
                             _p(codes), _p(sf), _p(D), _p(t))
    return codes, sf, np.float32(g[0]), t


# ---- O7/O8 forward --------------------------------------------------------

def linear_fwd_nvfp4(xc, xsf, g_x, wc, wsf, g_w, t, U_bits, M, N, K, rows=None):
    rows = _rows(rows, M)
    y = np.empty((len(rows), N), np.float64)
    xc, xsf, wc, wsf = (_c(a, np.uint8) for a in (xc, xsf, wc, wsf))
    t = None if t is None else _c(t, np.float64)
    U = None if U_bits is None else _c(U_bits, np.uint16)
    lib().or_linear_fwd_nvfp4(_p(xc), _p(xsf), float(g_x), _p(wc), _p(wsf), float(g_w),
                              _p(t), _p(U), M, N, K, _p(rows), len(rows), _p(y))
    return y


def linear_fwd_int4(xrot, codes, scales, t, U_bits, M, N, K, rows=None, group=32):
    rows = _rows(rows, M)
    y = np.empty((len(rows), N), np.float64)
    xrot = _c(xrot, np.float32)
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint16)
    t = None if t is None else _c(t, np.float64)
    U = None if U_bits is None else _c(U_bits, np.uint16)
    if group == 32:
        lib().or_linear_fwd_int4(_p(xrot), _p(codes), _p(scales), _p(t), _p(U), M, N, K,
                                 _p(rows), len(rows), _p(y))
    else:
        lib().or_linear_fwd_int4_g(_p(xrot), _p(codes), _p(scales), int(group), _p(t), _p(U), M, N, K,
                                   _p(rows), len(rows), _p(y))
    return y


# ---- v3.1 int8 per-row codec (rank-16 low-rank branch) ---------------------

RANK_INT8 = 16


def int8_row(r):
    """One rotated row (K % 256 == 0) -> (codes int8 [K], scale float32, winning j)."""
    r = _c(r, np.float32)
    K = r.shape[0]
    q = np.empty(K, np.int8)
    s = np.empty(1, np.float32)
    j = np.empty(1, np.uint8)
    lib().or_int8_row(_p(r), K, _p(q), _p(s), _p(j))
    return q, np.float32(s[0]), int(j[0])


def build_int8(R):
    """R [N, K] fp32 -> (codes int8 [N, K], scales float32 [N], frac uint8 [N])."""
    R = _c(R, np.float32)
    N, K = R.shape
    codes = np.empty((N, K), np.int8)
    scales = np.empty(N, np.float32)
    frac = np.empty(N, np.uint8)
    lib().or_build_int8(_p(R), N, K, _p(codes), _p(scales), _p(frac))
    return codes, scales, frac


def lowrank_input(x_bits, lora_down_bits):
    """t = x lora_down in fp64, [M, rank] (rank = lora_down's columns)."""
    x = _c(x_bits, np.uint16)
    D = _c(lora_down_bits, np.uint16)
    M, K = x.shape
    rank = D.shape[1]
    t = np.empty((M, rank), np.float64)
    lib().or_lowrank_input(_p(x), M, K, _p(D), rank, _p(t))
    return t


def linear_fwd_int8(xrot, codes, scales, t, U_bits, M, N, K, rows=None):
    """y rows of the int8 forward, fp64 [n_rows, N]; t [M, 16] fp64 and U [N, 16] bf16 bits, or None."""
    rows = _rows(rows, M)
    y = np.empty((len(rows), N), np.float64)
    t = None if t is None else _c(t, np.float64)
    U = None if U_bits is None else _c(U_bits, np.uint16)
    lib().or_linear_fwd_int8(_p(_c(xrot, np.float32)), _p(_c(codes, np.int8)), _p(_c(scales, np.float32)),
                             _p(t), _p(U), M, N, K, _p(rows), len(rows), _p(y))
    return y


# ---- O9 reconstruct -------------------------------------------------------

FMT_INT4 = 1
FMT_NVFP4 = 2
FMT_INT4_G64 = 3
FMT_INT8_ROW = 4


def reconstruct_bf16(fmt, codes, scales, g_w, U_bits, D_bits, N, K, residual_only=False):
    codes = _c(codes, np.int8 if fmt == FMT_INT8_ROW else np.uint8)
    scales = _c(scales, {FMT_NVFP4: np.uint8, FMT_INT8_ROW: np.float32}.get(fmt, np.uint16))
    U = _c(U_bits, np.uint16)
    D = _c(D_bits, np.uint16)
    W = np.empty((N, K), np.uint16)
    lib().or_reconstruct_bf16(int(fmt), _p(codes), _p(scales), float(np.float32(g_w)),
                              _p(U), _p(D), N, K, 1 if residual_only else 0, _p(W))
    return W


# ---- backward of the input ------------------------------------------------

def linear_bwd_dx(dy_bits, W_bits, rows=None):
    """dx = dy W in fp64 [n_rows, K]: dy [M, N] bf16 bits, W [N, K] bf16 bits (the reconstruct)."""
    dy = _c(dy_bits, np.uint16)
    W = _c(W_bits, np.uint16)
    M, N = dy.shape
    K = W.shape[1]
    rows = _rows(rows, M)
    dx = np.empty((len(rows), K), np.float64)
    lib().or_linear_bwd_dx(_p(dy), _p(W), M, N, K, _p(rows), len(rows), _p(dx))
    return dx


# ---- SVD init of the low-rank branch (SquareQ README, "Low-rank branch" paragraph) ----

def svd_residual(W, up_bits, down_bits):
    """R = RN(W - L), L the fmaf chain over the factors' rank (32, or 16 for the int8 mode) of bf16
    up [N, rank] and down [K, rank] (as the reconstruct)."""
    W = _c(W, np.float32)
    N, K = W.shape
    up = _c(up_bits, np.uint16)
    rank = up.shape[1]
    assert rank in (16, 32) and _c(down_bits, np.uint16).shape[1] == rank
    R = np.empty((N, K), np.float32)
    lib().or_svd_residual(_p(W), _p(up), _p(_c(down_bits, np.uint16)), N, K, rank, _p(R))
    return R


SVD_MAX_ITER = 500


def f64_to_bf16(v) -> int:
    """bf16 bits of a float64, rounded once (nearest, ties to even)."""
    return int(lib().or_f64_to_bf16(float(v)))


def svd_top(W, rank=32, max_iter=SVD_MAX_ITER):
    """Leading singular triplets of W [N, K] by the oracle's fp64 subspace iteration with a
    one-sided Jacobi Rayleigh-Ritz step (sq_oracle.c, or_svd_top) -> (sigma [rank], u [N, rank],
    v [K, rank], iterations)."""
    W = _c(W, np.float32)
    N, K = W.shape
    s = np.empty(rank, np.float64)
    u = np.empty((N, rank), np.float64)
    v = np.empty((K, rank), np.float64)
    it = lib().or_svd_top(_p(W), N, K, int(rank), int(max_iter), _p(s), _p(u), _p(v))
    return s, u, v, it


def svd_init(W, rank=32, max_iter=SVD_MAX_ITER):
    """Truncated SVD of W [N, K] in scalar C (sq_oracle.c, or_svd_init) ->
    (lora_up bf16 bits [N, rank], lora_down bf16 bits [K, rank], R fp32 [N, K], sigma fp64 [rank]).
    The singular values are split evenly: up = u sqrt(sigma), down = v sqrt(sigma), each rounded
    from fp64 to bf16 once (nearest, ties to even); R = RN(W - L) with the fmaf chain of
    svd_residual."""
    W = _c(W, np.float32)
    N, K = W.shape
    up = np.empty((N, rank), np.uint16)
    down = np.empty((K, rank), np.uint16)
    R = np.empty((N, K), np.float32)
    s = np.empty(rank, np.float64)
    lib().or_svd_init(_p(W), N, K, int(rank), int(max_iter), _p(up), _p(down), _p(R), _p(s))
    return up, down, R, s
