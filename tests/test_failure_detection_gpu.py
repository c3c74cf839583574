"""Failure detection on the GPU without a GPU fault (SquareQ README, "End-to-end": no
silent fallback; every wait in the library's kernels is bounded).

A kernel waits on a barrier that nothing arrives on, with a 20 ms limit: it must give
up, set the workspace status word and return normally; the host then reads
SQ_ERR_TIMEOUT through sq_check_device_status, the word is cleared, and the same
context runs a forward whose result still matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from sqcase import FWD_TOL, bf16_dev, host, norm_err, to_dev

pytestmark = pytest.mark.gpu

SQ_ERR_TIMEOUT = 8


def test_bounded_wait_reports_timeout_and_context_survives():
    import bit_quantized_frozen_b200 as sq
    assert torch.cuda.is_available()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    sq.sq_selftest_wait_timeout(ws, limit_us=20000)
    with pytest.raises(sq.SqError) as e:
        sq.sq_check_device_status(ws)
    assert e.value.status == SQ_ERR_TIMEOUT
    sq.sq_check_device_status(ws)                    # cleared by the read
    d = si.make_inputs(64, 512, 256, 71)
    w = sq.build_nvfp4(to_dev(d["R"]), bf16_dev(d["U"]), bf16_dev(d["D"]))
    y = sq.linear_fwd(w, bf16_dev(d["x"]))
    torch.cuda.synchronize()
    wc, wsf, gw = oracle.build_nvfp4(d["R"])
    xc, xsf, gx, t = oracle.act_quant_nvfp4(d["x"], d["D"])
    ref = oracle.linear_fwd_nvfp4(xc, xsf, gx, wc, wsf, gw, t, d["U"], 64, 256, 512)
    assert norm_err(host(y), ref) <= FWD_TOL


def test_library_status_word_clear_after_reconstruct():
    """sq_reconstruct_bf16 takes no workspace: its pipelined kernel reports a wait that gave up
    through the library's own status word, read with sq_check_device_status(NULL). After normal
    reconstructs (W and W^T) the word is clear."""
    import bit_quantized_frozen_b200 as sq
    assert torch.cuda.is_available()
    d = si.make_inputs(8, 512, 384, 72)
    w = sq.build_nvfp4(to_dev(d["R"]), bf16_dev(d["U"]), bf16_dev(d["D"]))
    sq.reconstruct_bf16(w)
    sq.reconstruct_bf16(w, transposed=True)
    torch.cuda.synchronize()
    sq.sq_check_device_status(None)


SQ_ERR_NONFINITE = 9


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")], ids=["nan", "inf", "-inf"])
def test_check_finite_flags_nonfinite_activation(bad):
    """SQ_CHECK_FINITE scans x before the forward: one NaN or infinity anywhere sets the
    workspace status word, read back as SQ_ERR_NONFINITE; a clean x, or the same x without the
    flag, leaves the word clear."""
    import bit_quantized_frozen_b200 as sq
    d = si.make_inputs(130, 512, 256, 73)
    w = sq.build_nvfp4(to_dev(d["R"]), bf16_dev(d["U"]), bf16_dev(d["D"]))
    ws = sq.workspace(sq.SQ_OP_LINEAR_FWD_NVFP4, 130, 256, 512)
    x = bf16_dev(d["x"])
    sq.linear_fwd(w, x, ws=ws, flags=sq.SQ_CHECK_FINITE)
    sq.sq_check_device_status(ws)                                    # clean input
    xb = x.clone()
    xb[129, 511] = bad                                               # the last value of a ragged M
    sq.linear_fwd(w, xb, ws=ws)
    sq.sq_check_device_status(ws)                                    # no scan without the flag
    sq.linear_fwd(w, xb, ws=ws, flags=sq.SQ_CHECK_FINITE)
    with pytest.raises(sq.SqError) as e:
        sq.sq_check_device_status(ws)
    assert e.value.status == SQ_ERR_NONFINITE
    # the int4 path and the activation quantisation entry take the flag too
    w4 = sq.build_int4(to_dev(d["R"]), bf16_dev(d["U"]), bf16_dev(d["D"]))
    ws4 = sq.workspace(sq.SQ_OP_LINEAR_FWD_INT4, 130, 256, 512)
    sq.linear_fwd(w4, xb, ws=ws4, flags=sq.SQ_CHECK_FINITE)
    with pytest.raises(sq.SqError) as e:
        sq.sq_check_device_status(ws4)
    assert e.value.status == SQ_ERR_NONFINITE
    wsa = sq.workspace(sq.SQ_OP_ACT_QUANT_NVFP4, 130, 0, 512)
    codes = torch.empty((130, 256), dtype=torch.uint8, device="cuda")
    sf = torch.empty(sq.sq_sf_bytes(130, 512), dtype=torch.uint8, device="cuda")
    gx = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.sq_act_quant_nvfp4(xb, codes, sf, gx, flags=sq.SQ_CHECK_FINITE, ws=wsa)
    with pytest.raises(sq.SqError) as e:
        sq.sq_check_device_status(wsa)
    assert e.value.status == SQ_ERR_NONFINITE
