"""The Python binding refuses a tensor too short for the call before anything reaches the library.

The C entry points take bare device pointers and cannot see where a buffer ends, so the binding
checks each tensor's byte count against what the call reads or writes through it (the shapes
that include/sq.h documents). Host logic only: CPU tensors of the right size get past the size
checks and stop at the binding's "expected a CUDA tensor", and one element fewer is refused with
the argument's name.
"""
import pytest
import torch

import bit_quantized_frozen_b200 as sq

N, K, M = 256, 512, 40


def t(shape, dtype):
    return torch.zeros(shape, dtype=dtype)


def short(x):
    """The same tensor, one element short."""
    return x.flatten()[:-1]


def expect(call, name):
    with pytest.raises(ValueError) as e:
        call()
    if name is None:
        assert "expected a CUDA tensor" in str(e.value), str(e.value)
    else:
        assert f"{name} holds" in str(e.value), str(e.value)


def check_each(fn, args, kwargs=None, skip=()):
    """fn(**args) passes the size checks; with any one tensor argument shortened it is refused."""
    kwargs = kwargs or {}
    expect(lambda: fn(**args, **kwargs), None)
    for name, v in args.items():
        if isinstance(v, torch.Tensor) and name not in skip:
            bad = dict(args, **{name: short(v)})
            expect(lambda: fn(**bad, **kwargs), name)


def weight(fmt):
    rank = sq.RANK_INT8 if fmt == sq.SQ_FMT_INT8_ROW else sq.RANK
    if fmt == sq.SQ_FMT_INT8_ROW:
        codes, scales, g = t((N, K), torch.int8), t(N, torch.float32), None
    elif fmt == sq.SQ_FMT_NVFP4:
        codes, scales, g = t((N, K // 2), torch.uint8), t(sq.sq_sf_bytes(N, K), torch.uint8), t(1, torch.float32)
    else:
        G = 64 if fmt == sq.SQ_FMT_INT4_G64 else 32
        codes, scales, g = t((N, K // 2), torch.uint8), t((N, K // G), torch.float16), None
    return sq.Weight(fmt, N, K, codes, scales, g, t((N, rank), torch.bfloat16), t((K, rank), torch.bfloat16))


FMTS = [sq.SQ_FMT_INT4_G32, sq.SQ_FMT_INT4_G64, sq.SQ_FMT_NVFP4, sq.SQ_FMT_INT8_ROW]


def test_builders():
    R = t((N, K), torch.float32)
    for group in (32, 64):
        check_each(lambda R, codes, scales, frac_idx: sq.sq_build_int4(R, codes, scales, frac_idx, group=group),
                   dict(R=R, codes=t((N, K // 2), torch.uint8), scales=t((N, K // group), torch.float16),
                        frac_idx=t((N, K // group), torch.uint8)), skip=("R",))
    check_each(sq.sq_build_int8, dict(R=R, codes=t((N, K), torch.int8), scales=t(N, torch.float32),
                                      frac_idx=t(N, torch.uint8)), skip=("R",))
    check_each(sq.sq_build_nvfp4, dict(R=R, codes=t((N, K // 2), torch.uint8),
                                       sf_tiled=t(sq.sq_sf_bytes(N, K), torch.uint8), g_w=t(1, torch.float32),
                                       ws=t(256, torch.uint8)), skip=("R", "ws"))
    # the shape comes from R itself, so R is refused only when its elements are too narrow
    expect(lambda: sq.sq_build_int8(t((N, K), torch.float16), t((N, K), torch.int8), t(N, torch.float32)), "R")


def test_svd_init():
    for rank in (32, 16):
        check_each(lambda W, omega, lora_up, lora_down, R: sq.sq_svd_init(W, omega, 4, lora_up, lora_down, R,
                                                                           t(256, torch.uint8)),
                   dict(W=t((N, K), torch.float32), omega=t((K, 32), torch.float32),
                        lora_up=t((N, rank), torch.bfloat16), lora_down=t((K, rank), torch.bfloat16),
                        R=t((N, K), torch.float32)), skip=("W", "lora_up"))


def test_act_quant():
    check_each(sq.sq_act_quant_nvfp4,
               dict(x=t((M, K), torch.bfloat16), codes=t((M, K // 2), torch.uint8),
                    sf_tiled=t(sq.sq_sf_bytes(M, K), torch.uint8), g_x=t(1, torch.float32),
                    lora_down=t((K, 32), torch.bfloat16), t=t((M, 32), torch.float32)), skip=("x",))


@pytest.mark.parametrize("fmt", FMTS)
def test_forward_reconstruct_backward(fmt):
    w = weight(fmt)
    for flags, ydt in ((0, torch.float32), (sq.SQ_OUT_BF16, torch.bfloat16)):
        check_each(lambda x, y, g_x: sq.sq_linear_fwd(w, x, y, g_x=g_x, flags=flags, ws=t(256, torch.uint8)),
                   dict(x=t((M, K), torch.bfloat16), y=t((M, N), ydt), g_x=t(1, torch.float32)), skip=("x",))
        check_each(lambda x, y: sq.sq_linear_fwd_noalloc(w, x, y, flags=flags),
                   dict(x=t((M, K), torch.bfloat16), y=t((M, N), ydt)), skip=("x",))
    # a float32 y is twice a bf16 one: a bf16-sized buffer without the flag is refused
    expect(lambda: sq.sq_linear_fwd(w, t((M, K), torch.bfloat16), t((M, N), torch.bfloat16)), "y")
    for transposed in (False, True):
        W = t((K, N) if transposed else (N, K), torch.bfloat16)
        check_each(lambda W_out: sq.sq_reconstruct_bf16(w, W_out), dict(W_out=W))
    check_each(lambda dy, dx: sq.sq_linear_bwd_dx(w, dy, dx, t(256, torch.uint8)),
               dict(dy=t((M, N), torch.bfloat16), dx=t((M, K), torch.float32)), skip=("dy",))


@pytest.mark.parametrize("fmt", FMTS)
def test_weight_fields(fmt):
    """Each payload field and low-rank factor of a Weight, one element short, is refused."""
    x, y = t((M, K), torch.bfloat16), t((M, N), torch.float32)
    expect(lambda: sq.sq_linear_fwd(weight(fmt), x, y), None)
    for field in ("codes", "scales", "g_w", "lora_up", "lora_down"):
        w = weight(fmt)
        if getattr(w, field) is None:
            continue
        setattr(w, field, short(getattr(w, field)))
        expect(lambda: sq.sq_linear_fwd(w, x, y), field)
        expect(lambda: sq.sq_reconstruct_bf16(w, t((N, K), torch.bfloat16)), field)
    w = weight(fmt)
    w.lora_up = w.lora_down = None                     # no low-rank term: NULL factors pass
    expect(lambda: sq.sq_linear_fwd(w, x, y), None)
