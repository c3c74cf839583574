"""The device-side index checks of the debug build (libsq_debug.so, SQ_DEBUG_CHECKS).

In that build the kernels that write the layer's outputs test each store's index against the
buffer before storing; a failed check skips the store and sets the status bit that
sq_check_device_status reports as SQ_ERR_INDEX -- nothing traps.  Checked here:
  - the debug library gives the same bits as the release library on every entry point of the
    tiny layer (builders, activation quantiser, forwards, reconstructs) and leaves every status
    word clean;
  - sq_selftest_index_check makes the check fail on purpose (an index one past its bound, never
    dereferenced): the host reads SQ_ERR_INDEX and the context then runs a forward that still
    matches the release library.
The debug library runs in a child process (the binding loads one library per process).
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import bit_quantized_frozen_b200 as sq
import synth_inputs as si
d = si.make_config("tiny_64x256x512")
bf = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
R, x, U, D = torch.from_numpy(d["R"]).cuda(), bf(d["x"]), bf(d["U"]), bf(d["D"])
M, K = x.shape
out = {"debug_checks": sq.sq_debug_checks()}
w4 = sq.build_int4(R, U, D)
w6 = sq.build_int4(R, U, D, group=64)
wn = sq.build_nvfp4(R, U, D)
w8 = sq.build_int8(R, U[:, :16].contiguous(), D[:, :16].contiguous())
codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
sf = torch.empty(sq.sq_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
gx = torch.empty(1, dtype=torch.float32, device="cuda")
t = torch.empty((M, 32), dtype=torch.float32, device="cuda")
ws = sq.workspace(sq.SQ_OP_ACT_QUANT_NVFP4, M, 0, K)
sq.sq_act_quant_nvfp4(x, codes, sf, gx, D, t, ws=ws)
res = {"int4": w4, "int4g64": w6, "nvfp4": wn, "int8": w8}
arrays = {}
for k, w in res.items():
    arrays[k + "_codes"] = w.codes
    arrays[k + "_scales"] = w.scales
    arrays[k + "_y"] = sq.linear_fwd(w, x)
    arrays[k + "_W"] = sq.reconstruct_bf16(w)
    arrays[k + "_Wres"] = sq.reconstruct_bf16(w, residual_only=True)
    arrays[k + "_Wt"] = sq.reconstruct_bf16(w, transposed=True)
arrays["act_codes"], arrays["act_sf"], arrays["act_t"] = codes, sf, t
torch.cuda.synchronize()
sq.sq_check_device_status(ws)
sq.sq_check_device_status(None)
status = {}
if len(sys.argv) > 3:
    sws = torch.zeros(64, dtype=torch.int32, device="cuda")
    sq.sq_selftest_index_check(sws)
    try:
        sq.sq_check_device_status(sws)
        status["selftest"] = "ok"
    except sq.SqError as e:
        status["selftest"] = sq.status_str(e.status)
    arrays["after_selftest_y"] = sq.linear_fwd(wn, x)
    torch.cuda.synchronize()
    sq.sq_check_device_status(None)
np.savez(sys.argv[2], **{k: v.contiguous().view(torch.uint8).cpu().numpy() for k, v in arrays.items()})
out.update(status)
print(json.dumps(out))
'''


def run_child(tmp_path, lib, tag, selftest=False):
    env = dict(os.environ)
    if lib:
        env["SQ_LIBSQ_PATH"] = lib
    path = str(tmp_path / f"{tag}.npz")
    args = [sys.executable, "-c", CHILD, ROOT, path] + (["selftest"] if selftest else [])
    p = subprocess.run(args, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-3000:]
    return json.loads(p.stdout.strip().splitlines()[-1]), dict(np.load(path))


def test_debug_build_matches_release_and_reports_index_errors(tmp_path):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_quantized_frozen_b200 import build as b
    dbg = b.build(debug_checks=True)
    info_r, rel = run_child(tmp_path, None, "release")
    info_d, deb = run_child(tmp_path, dbg, "debug", selftest=True)
    assert info_r["debug_checks"] == 0 and info_d["debug_checks"] == 1
    for k, v in rel.items():
        assert np.array_equal(v, deb[k]), f"{k} differs between the debug and the release library"
    assert info_d["selftest"] == "device index check failed"
    assert np.array_equal(deb["after_selftest_y"], rel["nvfp4_y"])
