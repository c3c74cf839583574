"""Per-operation timing of libsq on one GPU, for kernel work and ncu captures.

    python -m bit_quantized_frozen_b200.opbench [--config NAME] [--op OP ...]
                                                [--reps R] [--warmup W]

Builds one seeded synthetic layer (synth_inputs), then times each selected
operation alone with CUDA events on the launching stream, flushing L2 (a
256 MB write outside the events) before every call, and prints one JSON line
per operation: milliseconds (mean and min) and the algorithmic rate.  Every
call is the public C entry point with its normal arguments; nothing is
skipped.  `--reps 1 --warmup 0` gives exactly one launch sequence per op,
which is what an ncu capture of a single kernel wants.

Operations:
  act_quant            sq_act_quant_nvfp4 with the low-rank input t
  act_quant_nolowrank  sq_act_quant_nvfp4 without t (absmax pass + quantisation)
  fwd_nvfp4            sq_linear_fwd, NVFP4 weight
  fwd_int4             sq_linear_fwd, int4 group-32 weight
  fwd_int8             sq_linear_fwd, int8 per-row weight (rank-16 low-rank branch)
  build_nvfp4          sq_build_nvfp4
  build_int4           sq_build_int4, group 32
  build_int4_g64       sq_build_int4, group 64
  build_int8           sq_build_int8
  recon_nvfp4 / recon_int4 / recon_int4_g64 / recon_int8
                       sq_reconstruct_bf16 with the low-rank term
  recon_nvfp4_resid / recon_int4_resid / recon_int8_resid
                       sq_reconstruct_bf16 with SQ_RECON_RESIDUAL_ONLY
  recon_nvfp4_t        sq_reconstruct_bf16 with SQ_RECON_TRANSPOSED (W^T)
  bwd_dx_nvfp4         sq_linear_bwd_dx (transposed reconstruct + bf16 GEMM)
  svd_init             sq_svd_init (rank-32 SVD init, 8 rounds of subspace iteration)
                       of W = lora_up lora_down^T + R
  gemm_nvfp4 / gemm_int4 / gemm_bwd_dx
                       the tensor-core GEMM launch inside sq_linear_fwd /
                       sq_linear_bwd_dx, timed by the events the library records
                       around it (sq_set_gemm_events)

    python -m bit_quantized_frozen_b200.opbench --stack 28

times the builders on the builder stack of the down-projection shape instead: 28 residual
weights [6144, 16384] fp32 (seeds 4000 + i), each uploaded into one reused device buffer
(the upload untimed) and built with sq_build_int4 (group 32), sq_build_nvfp4 and
sq_build_int8; one JSON line per builder with the whole stack's algorithmic GB/s.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bit_quantized_frozen_b200 as sq  # noqa: E402
import synth_inputs as si  # noqa: E402

FLUSH_BYTES = 256 << 20

OPS = ["act_quant", "act_quant_nolowrank", "fwd_nvfp4", "fwd_int4", "fwd_int8", "build_nvfp4", "build_int4",
       "build_int4_g64", "build_int8", "recon_nvfp4", "recon_int4", "recon_int4_g64", "recon_int8",
       "recon_nvfp4_resid", "recon_int4_resid", "recon_int8_resid", "recon_nvfp4_t", "gemm_nvfp4", "gemm_int4",
       "bwd_dx_nvfp4", "gemm_bwd_dx", "svd_init"]
SVD_ITERS = 8


def work(op, M, N, K):
    """(unit, algorithmic amount per call): bytes moved at least once, or 2MNK flops."""
    NK, MK = N * K, M * K
    if op.startswith("act_quant"):
        return "GB/s", MK * (2 + 0.5 + 1 / 16) + (M * 32 * 4 if op == "act_quant" else 0)
    if op == "svd_init":   # fp32 FMA work: two products with W per round, then the residual's chain
        return "TFLOP/s", (4.0 * SVD_ITERS + 2.0) * N * K * 32
    if op.startswith("fwd") or op.startswith("gemm") or op.startswith("bwd"):
        return "TFLOP/s", 2.0 * M * N * K
    if op == "build_nvfp4":
        return "GB/s", NK * (4 + 0.5 + 1 / 16)
    if op == "build_int4":
        return "GB/s", NK * (4 + 0.5 + 3 / 32)
    if op == "build_int4_g64":
        return "GB/s", NK * (4 + 0.5 + 3 / 64)
    if op == "build_int8":
        return "GB/s", NK * (4 + 1) + N * 5
    if op.startswith("recon_int8"):
        return "GB/s", NK * (1 + 2) + N * 4
    scale = {"nvfp4": 1 / 16, "int4": 2 / 32, "int4_g64": 2 / 64}[
        op.split("_", 1)[1].replace("_resid", "").replace("_t", "")]
    return "GB/s", NK * (0.5 + scale + 2)


class Clocks:
    """nvidia-smi samples (SM MHz, power, throttle reasons) every 50 ms while running."""
    Q = ("clocks.sm,power.draw,clocks_event_reasons.sw_power_cap,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown")

    def __enter__(self):
        self.rows = []
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0],
                                       f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "50"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=lambda: [self.rows.append(ln) for ln in self.p.stdout], daemon=True)
            self.t.start()
            time.sleep(0.2)
        except OSError:
            self.p = None
        return self

    def __exit__(self, *exc):
        if self.p is not None:
            time.sleep(0.1)
            self.p.terminate()
            self.p.wait()

    def summary(self):
        vals = []
        for ln in self.rows:
            f = [x.strip() for x in ln.split(",")]
            try:
                vals.append((float(f[0]), float(f[1]), [n for n, v in zip(("sw_power_cap", "hw_slowdown",
                             "sw_thermal_slowdown"), f[2:]) if v.lower() == "active"]))
            except (ValueError, IndexError):
                pass
        if not vals:
            return None
        return {"sm_mhz_median": statistics.median(v[0] for v in vals), "sm_mhz_min": min(v[0] for v in vals),
                "power_w_max": max(v[1] for v in vals), "reasons": sorted({r for v in vals for r in v[2]}),
                "samples": len(vals)}


def run_stack(n_weights: int):
    """The builder stack: n residuals of the down-projection shape through one device buffer."""
    N, K = 6144, 16384
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    R = torch.empty((N, K), dtype=torch.float32, device=dev)
    host = torch.empty((N, K), dtype=torch.float32).pin_memory()
    c4 = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    s4 = torch.empty((N, K // 32), dtype=torch.float16, device=dev)
    f4 = torch.empty((N, K // 32), dtype=torch.uint8, device=dev)
    cn = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sfn = torch.empty(sq.sq_sf_bytes(N, K), dtype=torch.uint8, device=dev)
    gn = torch.empty(1, dtype=torch.float32, device=dev)
    ws_b = sq.workspace(sq.SQ_OP_BUILD_NVFP4, 0, N, K, dev)
    c8 = torch.empty((N, K), dtype=torch.int8, device=dev)
    s8 = torch.empty(N, dtype=torch.float32, device=dev)
    f8 = torch.empty(N, dtype=torch.uint8, device=dev)
    builders = {
        "build_int4": (lambda: sq.sq_build_int4(R, c4, s4, f4), N * K * (4 + 0.5 + 3 / 32)),
        "build_nvfp4": (lambda: sq.sq_build_nvfp4(R, cn, sfn, gn, ws_b), N * K * (4 + 0.5 + 1 / 16)),
        "build_int8": (lambda: sq.sq_build_int8(R, c8, s8, f8), N * K * (4 + 1) + N * 5),
    }
    ms = {k: [] for k in builders}
    for i in range(n_weights):
        host.copy_(torch.from_numpy(si.make_stack_residual(i, N, K)))
        R.copy_(host, non_blocking=True)                 # the upload is not timed
        torch.cuda.synchronize()
        if i == 0:                                       # one untimed pass: module load, attributes
            for fn, _ in builders.values():
                fn()
            torch.cuda.synchronize()
        evs = {}
        for k, (fn, _) in builders.items():
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            evs[k] = (a, b)
        torch.cuda.synchronize()
        for k, (a, b) in evs.items():
            ms[k].append(a.elapsed_time(b))
    for k, (_, nbytes) in builders.items():
        total = sum(ms[k])
        print(json.dumps({"op": k + "_stack", "weights": n_weights, "shape": [N, K], "ms_total": total,
                          "ms_per_weight_mean": statistics.mean(ms[k]), "ms_per_weight_max": max(ms[k]),
                          "GB/s": nbytes * n_weights / (total * 1e-3) / 1e9}), flush=True)


def main():
    p = argparse.ArgumentParser()
    p.add_argument("--config", default="large_4480x16384x6144", choices=sorted(si.CONFIGS))
    p.add_argument("--op", nargs="+", default=OPS, choices=OPS)
    p.add_argument("--reps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--clocks", action="store_true", help="sample SM clocks and power during the timed calls")
    p.add_argument("--stack", type=int, default=0, help="time the builders on this many stack weights instead")
    args = p.parse_args()
    if args.stack:
        run_stack(args.stack)
        return
    cfg = si.CONFIGS[args.config]
    M, N, K = cfg.M, cfg.N, cfg.K
    d = si.make_config(cfg.name)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    R = torch.from_numpy(d["R"]).to(dev)
    x, U, D = bf(d["x"]), bf(d["U"]), bf(d["D"])
    w4 = sq.build_int4(R, U, D)
    w6 = sq.build_int4(R, U, D, group=64)
    wn = sq.build_nvfp4(R, U, D)
    w8 = sq.build_int8(R, U[:, :16].contiguous(), D[:, :16].contiguous())
    ws_8 = sq.workspace(sq.SQ_OP_LINEAR_FWD_INT8, M, N, K, dev)
    ws_b = sq.workspace(sq.SQ_OP_BUILD_NVFP4, 0, N, K, dev)
    ws_a = sq.workspace(sq.SQ_OP_ACT_QUANT_NVFP4, M, 0, K, dev)
    ws_n = sq.workspace(sq.SQ_OP_LINEAR_FWD_NVFP4, M, N, K, dev)
    ws_i = sq.workspace(sq.SQ_OP_LINEAR_FWD_INT4, M, N, K, dev)
    xc = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    xsf = torch.empty(sq.sq_sf_bytes(M, K), dtype=torch.uint8, device=dev)
    gx = torch.empty(1, dtype=torch.float32, device=dev)
    t = torch.empty((M, 32), dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.float32, device=dev)
    W = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    Wt = torch.empty((K, N), dtype=torch.bfloat16, device=dev)
    dy = torch.randn((M, N), device=dev, generator=torch.Generator(device=dev).manual_seed(cfg.seed)).to(torch.bfloat16)
    dx = torch.empty((M, K), dtype=torch.float32, device=dev)
    ws_dx = sq.workspace(sq.SQ_OP_LINEAR_BWD_DX, M, N, K, dev)
    c4 = torch.empty_like(w4.codes)
    if "svd_init" in args.op:
        Wsvd = R + U.float() @ D.float().T
        omega = torch.randn((K, 32), device=dev, generator=torch.Generator(device=dev).manual_seed(cfg.seed))
        up_s = torch.empty((N, 32), dtype=torch.bfloat16, device=dev)
        down_s = torch.empty((K, 32), dtype=torch.bfloat16, device=dev)
        R_s = torch.empty_like(R)
        ws_s = sq.workspace(sq.SQ_OP_SVD_INIT, 0, N, K, dev)
    s4, f4 = torch.empty_like(w4.scales), torch.empty_like(w4.frac_idx)
    s6, f6 = torch.empty_like(w6.scales), torch.empty_like(w6.frac_idx)
    cn, sfn, gn = torch.empty_like(wn.codes), torch.empty_like(wn.scales), torch.empty_like(wn.g_w)
    c8, s8, f8 = torch.empty_like(w8.codes), torch.empty_like(w8.scales), torch.empty_like(w8.frac_idx)
    RES = sq.SQ_RECON_RESIDUAL_ONLY
    calls = {
        "act_quant": lambda: sq.sq_act_quant_nvfp4(x, xc, xsf, gx, D, t, ws=ws_a),
        "act_quant_nolowrank": lambda: sq.sq_act_quant_nvfp4(x, xc, xsf, gx, ws=ws_a),
        "fwd_nvfp4": lambda: sq.sq_linear_fwd(wn, x, y, g_x=gx, ws=ws_n),
        "fwd_int4": lambda: sq.sq_linear_fwd(w4, x, y, ws=ws_i),
        "fwd_int8": lambda: sq.sq_linear_fwd(w8, x, y, ws=ws_8),
        "build_int8": lambda: sq.sq_build_int8(R, c8, s8, f8),
        "recon_int8": lambda: sq.sq_reconstruct_bf16(w8, W),
        "recon_int8_resid": lambda: sq.sq_reconstruct_bf16(w8, W, RES),
        "build_nvfp4": lambda: sq.sq_build_nvfp4(R, cn, sfn, gn, ws_b),
        "build_int4": lambda: sq.sq_build_int4(R, c4, s4, f4),
        "build_int4_g64": lambda: sq.sq_build_int4(R, c4, s6, f6, group=64),
        "recon_nvfp4": lambda: sq.sq_reconstruct_bf16(wn, W),
        "recon_int4": lambda: sq.sq_reconstruct_bf16(w4, W),
        "recon_int4_g64": lambda: sq.sq_reconstruct_bf16(w6, W),
        "recon_nvfp4_resid": lambda: sq.sq_reconstruct_bf16(wn, W, RES),
        "recon_int4_resid": lambda: sq.sq_reconstruct_bf16(w4, W, RES),
        "recon_nvfp4_t": lambda: sq.sq_reconstruct_bf16(wn, Wt, sq.SQ_RECON_TRANSPOSED),
        "bwd_dx_nvfp4": lambda: sq.sq_linear_bwd_dx(wn, dy, dx, ws_dx),
        "gemm_bwd_dx": lambda: sq.sq_linear_bwd_dx(wn, dy, dx, ws_dx),
        "gemm_nvfp4": lambda: sq.sq_linear_fwd(wn, x, y, g_x=gx, ws=ws_n),
        "gemm_int4": lambda: sq.sq_linear_fwd(w4, x, y, ws=ws_i),
        "svd_init": lambda: sq.sq_svd_init(Wsvd, omega, SVD_ITERS, up_s, down_s, R_s, ws_s),
    }
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    for op in args.op:
        fn = calls[op]
        for _ in range(args.warmup):
            flush.fill_(1)
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.reps)]
        gemm = op.startswith("gemm")
        clk = Clocks() if args.clocks else None
        if clk:
            clk.__enter__()
        for a, b in evs:
            flush.fill_(1)
            if gemm:
                sq.sq_set_gemm_events(a, b)
            else:
                a.record()
            fn()
            if gemm:
                sq.sq_set_gemm_events(None, None)
            else:
                b.record()
        torch.cuda.synchronize()
        if clk:
            clk.__exit__(None, None, None)
        ms = [a.elapsed_time(b) for a, b in evs]
        unit, amount = work(op, M, N, K)
        rate = amount / (statistics.mean(ms) * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
        line = {"op": op, "config": cfg.name, "ms_mean": statistics.mean(ms), "ms_min": min(ms), unit: rate,
                "reps": args.reps}
        if clk:
            line["clocks"] = clk.summary()
        print(json.dumps(line), flush=True)
    sq.sq_check_device_status(ws_n)
    sq.sq_check_device_status(ws_i)


if __name__ == "__main__":
    main()
