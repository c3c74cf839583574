"""Python binding of libsq, the SquareQ W4 quantized linear layer for B200 (sm_100a).

Thin ctypes marshalling over the C ABI declared in ``include/sq.h``: every
function below has the same name as its C entry point, takes torch tensors
(device memory, contiguous) and passes their pointers, sizes and the current
CUDA stream.  All arithmetic runs in the library's CUDA kernels; there is no
CPU or PyTorch fallback -- if ``libsq.so`` is missing or the device is not
sm_100, the calls raise.

The layer (SquareQ README, section "SquareQ v3 -- W4"):
    W = lora_up @ lora_down^T + inverse_H256(dequant(residual))
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("SQ_LIBSQ_PATH") or os.path.join(_HERE, "libsq.so")

SQ_OK = 0
SQ_FMT_INT4_G32 = 1
SQ_FMT_NVFP4 = 2
SQ_FMT_INT4_G64 = 3
SQ_FMT_INT8_ROW = 4
SQ_OP_BUILD_INT4 = 1
SQ_OP_BUILD_NVFP4 = 2
SQ_OP_ACT_QUANT_NVFP4 = 3
SQ_OP_LINEAR_FWD_NVFP4 = 4
SQ_OP_LINEAR_FWD_INT4 = 5
SQ_OP_RECONSTRUCT = 6
SQ_OP_LINEAR_FWD_INT8 = 7
SQ_OP_BUILD_INT8 = 8
RANK_INT8 = 16
SQ_ACT_STATIC_SCALE = 0x1
SQ_RECON_RESIDUAL_ONLY = 0x2
SQ_RECON_TRANSPOSED = 0x4
SQ_OUT_BF16 = 0x8
SQ_STAGE_GEMM = 0                     # sq_set_stage_events
SQ_STAGE_ACT_PASS1 = 1
SQ_STAGE_ACT_QUANT = 2
SQ_CHECK_FINITE = 0x10
SQ_OP_LINEAR_BWD_DX = 9
SQ_OP_SVD_INIT = 10
RANK = 32

EXPORTED = [
    "sq_status_str", "sq_abi_version", "sq_debug_checks", "sq_selftest_index_check", "sq_last_error_detail", "sq_sf_bytes", "sq_workspace_bytes",
    "sq_build_int4", "sq_build_int8", "sq_build_nvfp4", "sq_act_quant_nvfp4", "sq_linear_fwd",
    "sq_reconstruct_bf16",
    "sq_check_device_status", "sq_set_gemm_events", "sq_set_stage_events", "sq_linear_fwd_noalloc", "sq_linear_bwd_dx",
    "sq_selftest_wait_timeout", "sq_svd_init",
]


class SqError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{fn} failed: {status_str(status)} ({status})"
        if detail:
            msg += f": {detail}"
        super().__init__(msg)


class sq_weight(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("N", ctypes.c_int64),
        ("K", ctypes.c_int64),
        ("codes", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("g_w", ctypes.c_void_p),
        ("lora_up", ctypes.c_void_p),
        ("lora_down", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGS = {
    "sq_status_str": ([ctypes.c_int], ctypes.c_char_p),
    "sq_abi_version": ([], ctypes.c_int),
    "sq_debug_checks": ([], ctypes.c_int),
    "sq_selftest_index_check": ([_P, _P], ctypes.c_int),
    "sq_last_error_detail": ([], ctypes.c_char_p),
    "sq_sf_bytes": ([_I64, _I64], ctypes.c_size_t),
    "sq_workspace_bytes": ([ctypes.c_int, _I64, _I64, _I64], ctypes.c_size_t),
    "sq_build_int4": ([_P, _I64, _I64, ctypes.c_int32, _P, _P, _P, _P], ctypes.c_int),
    "sq_build_int8": ([_P, _I64, _I64, _P, _P, _P, _P], ctypes.c_int),
    "sq_svd_init": ([_P, _I64, _I64, _P, ctypes.c_int32, ctypes.c_int32, _P, _P, _P, _P, ctypes.c_size_t, _P],
                    ctypes.c_int),
    "sq_build_nvfp4": ([_P, _I64, _I64, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "sq_act_quant_nvfp4": ([_P, _I64, _I64, _P, _P, _P, _P, _P, ctypes.c_uint32, _P, ctypes.c_size_t, _P],
                           ctypes.c_int),
    "sq_linear_fwd": ([ctypes.POINTER(sq_weight), _P, _I64, _P, _P, ctypes.c_uint32, _P, ctypes.c_size_t, _P],
                      ctypes.c_int),
    "sq_linear_fwd_noalloc": ([ctypes.POINTER(sq_weight), _P, _I64, _P, _P, ctypes.c_uint32,
                               ctypes.POINTER(ctypes.c_void_p), _P], ctypes.c_int),
    "sq_reconstruct_bf16": ([ctypes.POINTER(sq_weight), _P, ctypes.c_uint32, _P], ctypes.c_int),
    "sq_linear_bwd_dx": ([ctypes.POINTER(sq_weight), _P, _I64, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "sq_check_device_status": ([_P, _P], ctypes.c_int),
    "sq_selftest_wait_timeout": ([_P, ctypes.c_uint32, _P], ctypes.c_int),
    "sq_set_gemm_events": ([_P, _P], ctypes.c_int),
    "sq_set_stage_events": ([ctypes.c_int32, _P, _P], ctypes.c_int),
}
_lib = None


def lib() -> ctypes.CDLL:
    """Load libsq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libsq.so not found at {LIB_PATH}; build it with "
                               "`python -m bit_quantized_frozen_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().sq_status_str(int(status)).decode()


def _check(fn: str, status: int):
    if status != SQ_OK:
        raise SqError(fn, status, lib().sq_last_error_detail().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _numel_bytes(t) -> int:
    return t.numel() * t.element_size()


def _need(fn: str, name: str, t, nbytes: int):
    """Raise before the call if tensor t holds fewer bytes than the entry point reads or writes
    through it.  The C entry points take bare pointers and cannot see a buffer's end, so a short
    tensor would be overrun on the device.  None (a NULL argument) and raw integer addresses are
    passed through unchecked; the library validates the rest (shapes, alignment, flags)."""
    if t is None or isinstance(t, int):
        return
    have = _numel_bytes(t)
    if have < nbytes:
        raise ValueError(f"{fn}: {name} holds {have} bytes, the call needs {nbytes}")


def _need_weight(fn: str, w: "Weight"):
    """The payload and low-rank factors of a built weight, sized by its format."""
    N, K = int(w.N), int(w.K)
    if N <= 0 or K <= 0:
        return                                   # the library rejects the shape
    if w.fmt == SQ_FMT_INT8_ROW:
        _need(fn, "codes", w.codes, N * K)
        _need(fn, "scales", w.scales, 4 * N)
        rank = RANK_INT8
    else:
        _need(fn, "codes", w.codes, N * K // 2)
        if w.fmt == SQ_FMT_NVFP4:
            _need(fn, "scales", w.scales, sq_sf_bytes(N, K))
            _need(fn, "g_w", w.g_w, 4)
        elif w.fmt in (SQ_FMT_INT4_G32, SQ_FMT_INT4_G64):
            _need(fn, "scales", w.scales, 2 * N * (K // (64 if w.fmt == SQ_FMT_INT4_G64 else 32)))
        rank = RANK
    _need(fn, "lora_up", w.lora_up, 2 * N * rank)
    _need(fn, "lora_down", w.lora_down, 2 * K * rank)


# ---- C entry points ----------------------------------------------------------

def sq_abi_version() -> int:
    return lib().sq_abi_version()


def sq_sf_bytes(rows: int, K: int) -> int:
    return lib().sq_sf_bytes(rows, K)


def sq_workspace_bytes(op: int, M: int, N: int, K: int) -> int:
    return lib().sq_workspace_bytes(op, M, N, K)


def sq_build_int4(R, codes, scales, frac_idx=None, group: int = 32, stream=None):
    N, K = R.shape
    if group in (32, 64):
        fn, G = "sq_build_int4", N * (K // group)
        _need(fn, "R", R, 4 * N * K)
        _need(fn, "codes", codes, N * K // 2)
        _need(fn, "scales", scales, 2 * G)
        _need(fn, "frac_idx", frac_idx, G)
    _check("sq_build_int4", lib().sq_build_int4(_ptr(R), N, K, group, _ptr(codes), _ptr(scales), _ptr(frac_idx),
                                                _stream(stream)))


def sq_svd_init(W, omega, iters, lora_up, lora_down, R, ws, stream=None):
    """The rank (32 or 16) is lora_up's number of columns."""
    N, K = W.shape
    rank = int(lora_up.shape[1])
    fn = "sq_svd_init"
    _need(fn, "W", W, 4 * N * K)
    _need(fn, "omega", omega, 4 * K * RANK)
    _need(fn, "lora_up", lora_up, 2 * N * rank)
    _need(fn, "lora_down", lora_down, 2 * K * rank)
    _need(fn, "R", R, 4 * N * K)
    _check("sq_svd_init", lib().sq_svd_init(_ptr(W), N, K, _ptr(omega), int(iters), rank, _ptr(lora_up),
                                            _ptr(lora_down), _ptr(R), _ptr(ws), _numel_bytes(ws), _stream(stream)))


def sq_build_int8(R, codes, scales, frac_idx=None, stream=None):
    N, K = R.shape
    fn = "sq_build_int8"
    _need(fn, "R", R, 4 * N * K)
    _need(fn, "codes", codes, N * K)
    _need(fn, "scales", scales, 4 * N)
    _need(fn, "frac_idx", frac_idx, N)
    _check("sq_build_int8", lib().sq_build_int8(_ptr(R), N, K, _ptr(codes), _ptr(scales), _ptr(frac_idx),
                                                _stream(stream)))


def sq_build_nvfp4(R, codes, sf_tiled, g_w, ws, stream=None):
    N, K = R.shape
    fn = "sq_build_nvfp4"
    _need(fn, "R", R, 4 * N * K)
    _need(fn, "codes", codes, N * K // 2)
    _need(fn, "sf_tiled", sf_tiled, sq_sf_bytes(N, K) if N > 0 and K > 0 else 0)
    _need(fn, "g_w", g_w, 4)
    _check("sq_build_nvfp4", lib().sq_build_nvfp4(_ptr(R), N, K, _ptr(codes), _ptr(sf_tiled), _ptr(g_w), _ptr(ws),
                                                  _numel_bytes(ws), _stream(stream)))


def sq_act_quant_nvfp4(x, codes, sf_tiled, g_x, lora_down=None, t=None, flags: int = 0, ws=None, stream=None):
    M, K = x.shape
    fn = "sq_act_quant_nvfp4"
    _need(fn, "x", x, 2 * M * K)
    _need(fn, "codes", codes, M * K // 2)
    _need(fn, "sf_tiled", sf_tiled, sq_sf_bytes(M, K) if M > 0 and K > 0 else 0)
    _need(fn, "g_x", g_x, 4)
    if lora_down is not None and t is not None:
        _need(fn, "lora_down", lora_down, 2 * K * RANK)
        _need(fn, "t", t, 4 * M * RANK)
    _check("sq_act_quant_nvfp4",
           lib().sq_act_quant_nvfp4(_ptr(x), M, K, _ptr(codes), _ptr(sf_tiled), _ptr(g_x), _ptr(lora_down), _ptr(t),
                                    flags, _ptr(ws), 0 if ws is None else _numel_bytes(ws), _stream(stream)))


def _need_fwd(fn: str, w: "Weight", x, y, g_x, flags: int):
    M = x.shape[0]
    _need_weight(fn, w)
    _need(fn, "x", x, 2 * M * int(w.K))
    _need(fn, "y", y, M * int(w.N) * (2 if flags & SQ_OUT_BF16 else 4))
    _need(fn, "g_x", g_x, 4)


def sq_linear_fwd(w: "Weight", x, y, g_x=None, flags: int = 0, ws=None, stream=None):
    M = x.shape[0]
    _need_fwd("sq_linear_fwd", w, x, y, g_x, flags)
    cw = w.as_c()
    _check("sq_linear_fwd", lib().sq_linear_fwd(ctypes.byref(cw), _ptr(x), M, _ptr(y), _ptr(g_x), flags, _ptr(ws),
                                                0 if ws is None else _numel_bytes(ws), _stream(stream)))


def sq_linear_fwd_noalloc(w: "Weight", x, y, g_x=None, flags: int = 0, stream=None) -> int:
    """sq_linear_fwd on libsq's static per-device scratch (no workspace);
    returns the scratch's device address (for sq_check_device_status)."""
    M = x.shape[0]
    _need_fwd("sq_linear_fwd_noalloc", w, x, y, g_x, flags)
    cw = w.as_c()
    scratch = ctypes.c_void_p()
    _check("sq_linear_fwd_noalloc", lib().sq_linear_fwd_noalloc(ctypes.byref(cw), _ptr(x), M, _ptr(y), _ptr(g_x),
                                                                flags, ctypes.byref(scratch), _stream(stream)))
    return scratch.value


def sq_reconstruct_bf16(w: "Weight", W_out, flags: int = 0, stream=None):
    _need_weight("sq_reconstruct_bf16", w)
    _need("sq_reconstruct_bf16", "W_out", W_out, 2 * int(w.N) * int(w.K))
    cw = w.as_c()
    _check("sq_reconstruct_bf16", lib().sq_reconstruct_bf16(ctypes.byref(cw), _ptr(W_out), flags, _stream(stream)))


def sq_linear_bwd_dx(w: "Weight", dy, dx, ws, stream=None):
    M = dy.shape[0]
    fn = "sq_linear_bwd_dx"
    _need_weight(fn, w)
    _need(fn, "dy", dy, 2 * M * int(w.N))
    _need(fn, "dx", dx, 4 * M * int(w.K))
    cw = w.as_c()
    _check("sq_linear_bwd_dx", lib().sq_linear_bwd_dx(ctypes.byref(cw), _ptr(dy), M, _ptr(dx), _ptr(ws),
                                                      _numel_bytes(ws), _stream(stream)))


def sq_debug_checks() -> int:
    """1 if the loaded library was built with the device-side index checks (libsq_debug.so)."""
    return lib().sq_debug_checks()


def sq_selftest_index_check(ws, stream=None):
    _check("sq_selftest_index_check", lib().sq_selftest_index_check(_ptr(ws), _stream(stream)))


def sq_selftest_wait_timeout(ws, limit_us: int = 20000, stream=None):
    _check("sq_selftest_wait_timeout", lib().sq_selftest_wait_timeout(_ptr(ws), int(limit_us), _stream(stream)))


def sq_check_device_status(ws, stream=None):
    _check("sq_check_device_status", lib().sq_check_device_status(_ptr(ws), _stream(stream)))


def _event_handle(ev):
    if ev is None:
        return None
    if ev.cuda_event == 0:              # torch creates the CUDA event lazily
        ev.record()
    return ev.cuda_event


def sq_set_gemm_events(start_event=None, stop_event=None):
    """Record these torch.cuda.Event objects around the GEMM launch of later
    sq_linear_fwd calls on this thread (None, None turns it off)."""
    _check("sq_set_gemm_events", lib().sq_set_gemm_events(_event_handle(start_event), _event_handle(stop_event)))


def sq_set_stage_events(stage: int, start_event=None, stop_event=None):
    """The same for SQ_STAGE_GEMM, SQ_STAGE_ACT_PASS1 or SQ_STAGE_ACT_QUANT."""
    _check("sq_set_stage_events",
           lib().sq_set_stage_events(int(stage), _event_handle(start_event), _event_handle(stop_event)))


# ---- a built weight and allocating helpers (torch provides the memory) --------

@dataclass
class Weight:
    fmt: int
    N: int
    K: int
    codes: torch.Tensor                  # uint8 [N, K/2] (int8 format: int8 [N, K])
    scales: torch.Tensor                 # int4: float16 [N, K/group]; NVFP4: uint8 tiled; int8: float32 [N]
    g_w: torch.Tensor | None = None      # float32 [1] (NVFP4)
    lora_up: torch.Tensor | None = None  # bf16 [N, 32] (int8 format: [N, 16])
    lora_down: torch.Tensor | None = None  # bf16 [K, 32] (int8 format: [K, 16])
    frac_idx: torch.Tensor | None = None  # uint8 [N, K/group] (int4), [N] (int8)

    def as_c(self) -> sq_weight:
        return sq_weight(self.fmt, self.N, self.K, _ptr(self.codes), _ptr(self.scales), _ptr(self.g_w),
                         _ptr(self.lora_up), _ptr(self.lora_down))


def workspace(op: int, M: int, N: int, K: int, device=None) -> torch.Tensor:
    n = max(sq_workspace_bytes(op, M, N, K), 256)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def build_int4(R: torch.Tensor, lora_up=None, lora_down=None, group: int = 32, stream=None) -> Weight:
    N, K = R.shape
    dev = R.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    frac = torch.empty((N, K // group), dtype=torch.uint8, device=dev)
    sq_build_int4(R, codes, scales, frac, group=group, stream=stream)
    fmt = SQ_FMT_INT4_G64 if group == 64 else SQ_FMT_INT4_G32
    return Weight(fmt, N, K, codes, scales, None, lora_up, lora_down, frac)


def build_int8(R: torch.Tensor, lora_up=None, lora_down=None, stream=None) -> Weight:
    """int8 per-row weight; lora_up [N, 16] / lora_down [K, 16] (rank 16) or None."""
    N, K = R.shape
    dev = R.device
    codes = torch.empty((N, K), dtype=torch.int8, device=dev)
    scales = torch.empty(N, dtype=torch.float32, device=dev)
    frac = torch.empty(N, dtype=torch.uint8, device=dev)
    sq_build_int8(R, codes, scales, frac, stream=stream)
    return Weight(SQ_FMT_INT8_ROW, N, K, codes, scales, None, lora_up, lora_down, frac)


def build_nvfp4(R: torch.Tensor, lora_up=None, lora_down=None, ws=None, stream=None) -> Weight:
    N, K = R.shape
    dev = R.device
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sf = torch.empty(sq_sf_bytes(N, K), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    ws = ws if ws is not None else workspace(SQ_OP_BUILD_NVFP4, 0, N, K, dev)
    sq_build_nvfp4(R, codes, sf, g, ws, stream=stream)
    return Weight(SQ_FMT_NVFP4, N, K, codes, sf, g, lora_up, lora_down)


def svd_init(W: torch.Tensor, omega: torch.Tensor, iters: int = 8, rank: int = RANK, stream=None):
    """(lora_up bf16 [N, rank], lora_down bf16 [K, rank], R fp32 [N, K]) of W [N, K] fp32; rank 32,
    or 16 (RANK_INT8) for the int8 mode."""
    N, K = W.shape
    dev = W.device
    up = torch.empty((N, rank), dtype=torch.bfloat16, device=dev)
    down = torch.empty((K, rank), dtype=torch.bfloat16, device=dev)
    R = torch.empty((N, K), dtype=torch.float32, device=dev)
    ws = workspace(SQ_OP_SVD_INIT, 0, N, K, dev)
    sq_svd_init(W, omega, iters, up, down, R, ws, stream=stream)
    return up, down, R


def linear_fwd(w: Weight, x: torch.Tensor, ws=None, g_x=None, flags: int = 0, out_bf16: bool = False,
               stream=None) -> torch.Tensor:
    """y [M, N] = x W^T: fp32, or bf16 (the same values rounded once) with out_bf16."""
    M = x.shape[0]
    if out_bf16:
        flags |= SQ_OUT_BF16
    y = torch.empty((M, w.N), dtype=torch.bfloat16 if flags & SQ_OUT_BF16 else torch.float32, device=x.device)
    op = {SQ_FMT_NVFP4: SQ_OP_LINEAR_FWD_NVFP4, SQ_FMT_INT8_ROW: SQ_OP_LINEAR_FWD_INT8}.get(w.fmt, SQ_OP_LINEAR_FWD_INT4)
    ws = ws if ws is not None else workspace(op, M, w.N, w.K, x.device)
    sq_linear_fwd(w, x, y, g_x=g_x, flags=flags, ws=ws, stream=stream)
    return y


def reconstruct_bf16(w: Weight, residual_only: bool = False, transposed: bool = False, stream=None) -> torch.Tensor:
    shape = (w.K, w.N) if transposed else (w.N, w.K)
    W = torch.empty(shape, dtype=torch.bfloat16, device=w.codes.device)
    flags = (SQ_RECON_RESIDUAL_ONLY if residual_only else 0) | (SQ_RECON_TRANSPOSED if transposed else 0)
    sq_reconstruct_bf16(w, W, flags, stream=stream)
    return W


def linear_bwd_dx(w: Weight, dy: torch.Tensor, ws=None, stream=None) -> torch.Tensor:
    """dx = dy W (dy [M, N] bf16) as fp32 [M, K]."""
    M = dy.shape[0]
    dx = torch.empty((M, w.K), dtype=torch.float32, device=dy.device)
    ws = ws if ws is not None else workspace(SQ_OP_LINEAR_BWD_DX, M, w.N, w.K, dy.device)
    sq_linear_bwd_dx(w, dy, dx, ws, stream=stream)
    return dx
