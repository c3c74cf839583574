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
