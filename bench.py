#!/usr/bin/env python
"""Benchmark of the SquareQ W4 linear layer hot path on B200.

One step = one pass of the whole hot path over one synthetic layer of the
chosen shape (default the headline 4480 x 16384 x 6144, M x N x K):
  sq_build_int4, sq_build_nvfp4, sq_linear_fwd (NVFP4, incl. the activation
  prologue; fp32 y, and bf16 y with SQ_OUT_BF16), sq_linear_fwd (int4), sq_reconstruct_bf16 (both payloads), and the
  build, forward and reconstruct of the int4 group-64 variant and of the int8
  per-row mode (rank-16 low-rank branch), the input backward dx = dy W
  (transposed bf16 reconstruct + bf16 GEMM) on the NVFP4 payload, and the
  rank-32 SVD init of W = lora_up lora_down^T + R (sq_svd_init, 8 rounds).
Every op is timed with CUDA events on the launching stream after an L2 flush
(a 256 MB write outside the op's events); the NVFP4 forward is the headline
metric (TFLOP/s = 2 M N K / time of the whole sq_linear_fwd call).  The GEMM
kernel alone is timed with events recorded around its launch inside the
library (sq_set_gemm_events) for the roofline line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica (the layer does not shard; no collective on the data path) and the
device time is the max over ranks.  --impl reference times the CPU oracle on a
bounded sample of the same workload on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402

METRIC = "W4 linear fwd TFLOP/s & % FP4/BF16 tensor peak; quantize/reconstruct GB/s % HBM"
HEADLINE = "large_4480x16384x6144"
# SquareQ README, NVFP4 vs bf16 table: 4480 x 16384 x 6144 fp4 GEMM 1074 us on an
# RTX 5080 (sm_120, cuBLASLt), i.e. 2*4480*16384*6144 / 1074e-6 = 840.3 TFLOP/s.
PAGES_FP4_TFLOPS = {"large_4480x16384x6144": 2 * 4480 * 16384 * 6144 / 1074e-6 / 1e12}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_PER_BF16 = 4.0        # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
FLUSH_BYTES = 256 << 20   # > 126 MB L2
# FP32 FMA issue roofline of the SVD init's products: 148 SMs x 128 FMA lanes x 2 flop x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
ALU_GOPS = 148 * 128 * 1.965e9 / 1e9    # FP32 lane-operations per second at the maximum SM clock
# algorithmic FP32 lane-operations per element of the [N, K] operand for the ALU-bound kernels:
# the builders' 26-trial sweep (multiply, round, clamp, error, square, sum: 8 per trial) plus the
# Hadamard transform (8), the reconstruct's rank-r fmaf chain plus the transform
ALU_OPS = {"build_int4": 26 * 8 + 8, "build_int4_g64": 26 * 8 + 8, "build_int8": 26 * 8 + 8,
           "reconstruct_nvfp4": 32 + 8, "reconstruct_int4": 32 + 8, "reconstruct_int4_g64": 32 + 8,
           "reconstruct_int8": 16 + 8}
SVD_ITERS = 8


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="sq", choices=["sq", "reference"])
    p.add_argument("--config", default=HEADLINE, choices=sorted(si.CONFIGS))
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--no-extra", action="store_true", help="skip the other configurations and the builder stack")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# per-op algorithmic work (bytes per element of the [N,K] or [M,K] operand)
# ---------------------------------------------------------------------------

def op_work(M, N, K):
    NK, MK = N * K, M * K
    return {
        "build_int4": ("GB/s", NK * (4 + 0.5 + 2 / 32 + 1 / 32)),
        "build_nvfp4": ("GB/s", NK * (4 + 0.5 + 1 / 16)),
        "fwd_nvfp4": ("TFLOP/s", 2.0 * M * N * K),
        "fwd_nvfp4_bf16out": ("TFLOP/s", 2.0 * M * N * K),
        "fwd_int4": ("TFLOP/s", 2.0 * M * N * K),
        "reconstruct_nvfp4": ("GB/s", NK * (0.5 + 1 / 16 + 2)),
        "reconstruct_int4": ("GB/s", NK * (0.5 + 2 / 32 + 2)),
        "build_int4_g64": ("GB/s", NK * (4 + 0.5 + 2 / 64 + 1 / 64)),
        "fwd_int4_g64": ("TFLOP/s", 2.0 * M * N * K),
        "reconstruct_int4_g64": ("GB/s", NK * (0.5 + 2 / 64 + 2)),
        "build_int8": ("GB/s", NK * (4 + 1) + N * 5),
        "fwd_int8": ("TFLOP/s", 2.0 * M * N * K),
        "reconstruct_int8": ("GB/s", NK * (1 + 2) + N * 4),
        "bwd_dx_nvfp4": ("TFLOP/s", 2.0 * M * N * K),
        "svd_init": ("TFLOP/s", (4.0 * SVD_ITERS + 2.0) * NK * 32),   # fp32 FMA work (2 products/round + residual)
        "act_quant_nvfp4": ("GB/s", MK * (2 + 0.5 + 1 / 16) + M * 32 * 4),
        "act_pass1": ("GB/s", MK * 2 + M * 32 * 4),            # x read once (absmax and t)
        "act_pass2": ("GB/s", MK * (2 + 0.5 + 1 / 16)),        # x again, codes and scales
        "reconstruct_nvfp4_resid": ("GB/s", NK * (0.5 + 1 / 16 + 2)),
        "gemm_nvfp4": ("TFLOP/s", 2.0 * M * N * K),
        "gemm_int4": ("TFLOP/s", 2.0 * M * N * K),
        "gemm_bwd_dx": ("TFLOP/s", 2.0 * M * N * K),
    }


LAUNCHES_PER_STEP = {   # our kernels per op (memsets excluded)
    "build_int4": 1, "build_nvfp4": 2, "fwd_nvfp4": 3, "fwd_nvfp4_bf16out": 3, "fwd_int4": 5,
    "act_quant_nvfp4": 2, "reconstruct_nvfp4_resid": 1,
    "reconstruct_nvfp4": 1, "reconstruct_int4": 1,
    "build_int4_g64": 1, "fwd_int4_g64": 5, "reconstruct_int4_g64": 1,
    "build_int8": 1, "fwd_int8": 7, "reconstruct_int8": 1,
    "bwd_dx_nvfp4": 2,
    # start block orth (3) + per round: 2 products, 2 split sums, orth(U) and orth(V) of 3 kernels
    # per pass (one pass each; the last round two for U and none for V) + Gram, Jacobi, factors,
    # residual
    "svd_init": 3 + 10 * SVD_ITERS + 4,
}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:7], float(parts[7])))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r[3] > 0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len([r for r in rows if r[3] > 0])}


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# ---------------------------------------------------------------------------
# roofline traffic from the committed ncu summary (null once the kernel changed)
# ---------------------------------------------------------------------------

GEMM_SOURCES = ["bit_quantized_frozen_b200/csrc/sq_gemm.cu", "bit_quantized_frozen_b200/csrc/sq_ptx.cuh"]


def code_only(text: str) -> str:
    """C/C++ source without its comments, trailing blanks and empty lines."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def gemm_source_hash(read=None) -> str:
    """First 16 hex digits of sha256 over the GEMM's sources with comments removed: an edit of a
    comment keeps the ncu counters, any change of code drops them.  read(rel) returns a source's
    text (default: the file in this tree)."""
    read = read or (lambda rel: open(os.path.join(ROOT, rel)).read())
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        h.update(code_only(read(rel)).encode())
    return h.hexdigest()[:16]


def profiled_traffic(config: str):
    """dram bytes per launch of the NVFP4 GEMM from profiles/, scaled to `config`."""
    path = os.path.join(ROOT, "profiles", "gemm_nvfp4_4480x16384x6144.md")
    if not os.path.exists(path):
        return None, "no ncu summary"
    text = open(path).read()
    m_hash = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    if not m_hash or m_hash.group(1) != gemm_source_hash():
        return None, "kernel changed since the ncu capture"
    m = re.search(rf"traffic_bytes_per_launch\[{re.escape(config)}\]:\s*([0-9.eE+]+)", text)
    if not m:
        return None, "no capture for this workload"
    return float(m.group(1)), "ncu"


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------

def cpu_sample(d, M_s: int, N_s: int):
    """Run the oracle's whole pipeline on rows [0, N_s) of R and [0, M_s) of x.
    Returns per-op seconds."""
    import oracle
    oracle.build()
    R = np.ascontiguousarray(d["R"][:N_s])
    x = np.ascontiguousarray(d["x"][:M_s])
    U = np.ascontiguousarray(d["U"][:N_s])
    D = d["D"]
    K = R.shape[1]
    t = {}
    t0 = time.perf_counter()
    c4, s4, _ = oracle.build_int4(R)
    t["build_int4"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    wc, wsf, gw = oracle.build_nvfp4(R)
    t["build_nvfp4"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    xc, xsf, gx, tt = oracle.act_quant_nvfp4(x, D)
    oracle.linear_fwd_nvfp4(xc, xsf, gx, wc, wsf, gw, tt, U, M_s, N_s, K)
    t["fwd_nvfp4"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    xr = oracle.rotate_rows_bf16(x)
    _, _, _, tt2 = oracle.act_quant_nvfp4(x, D)
    oracle.linear_fwd_int4(xr, c4, s4, tt2, U, M_s, N_s, K)
    t["fwd_int4"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.reconstruct_bf16(2, wc, wsf, gw, U, D, N_s, K)
    t["reconstruct_nvfp4"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.reconstruct_bf16(1, c4, s4, 0.0, U, D, N_s, K)
    t["reconstruct_int4"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    c6, s6, _ = oracle.build_int4(R, group=64)
    t["build_int4_g64"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    xr = oracle.rotate_rows_bf16(x)
    _, _, _, tt3 = oracle.act_quant_nvfp4(x, D)
    oracle.linear_fwd_int4(xr, c6, s6, tt3, U, M_s, N_s, K, group=64)
    t["fwd_int4_g64"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.reconstruct_bf16(oracle.FMT_INT4_G64, c6, s6, 0.0, U, D, N_s, K)
    t["reconstruct_int4_g64"] = time.perf_counter() - t0
    U16, D16 = np.ascontiguousarray(U[:, :16]), np.ascontiguousarray(D[:, :16])
    t0 = time.perf_counter()
    c8, s8, _ = oracle.build_int8(R)
    t["build_int8"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    xr = oracle.rotate_rows_bf16(x)
    tt4 = oracle.lowrank_input(x, D16)
    oracle.linear_fwd_int8(xr, c8, s8, tt4, U16, M_s, N_s, K)
    t["fwd_int8"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.reconstruct_bf16(oracle.FMT_INT8_ROW, c8, s8, 0.0, U16, D16, N_s, K)
    t["reconstruct_int8"] = time.perf_counter() - t0
    n_svd = min(N_s, SVD_SAMPLE_ROWS)
    Wsvd = (R[:n_svd].astype(np.float64) + si.bf16_bits_to_f32(U[:n_svd]).astype(np.float64)
            @ si.bf16_bits_to_f32(D).astype(np.float64).T).astype(np.float32)
    t0 = time.perf_counter()
    oracle.svd_init(Wsvd)
    t["svd_init"] = time.perf_counter() - t0
    return t, oracle.num_threads()


SVD_SAMPLE_ROWS = 64       # the oracle's SVD init runs on the first 64 rows of W (its 64-vector
                           # subspace then spans the sample's row space: two rounds)
REF_SAMPLE = (64, 2048)    # reference arm, per step: M_s rows of x, N_s rows of R (all K)
CPU_SAMPLE = (128, 4096)   # one-off CPU baseline of the GPU arm


def cpu_sample_desc(cfg, M_s, N_s):
    return (f"oracle pipeline on x rows 0..{M_s - 1} and R rows 0..{N_s - 1} (all K={cfg.K}) of the "
            f"{cfg.M}x{cfg.N}x{cfg.K} workload; metric = 2*{M_s}*{N_s}*{cfg.K} / oracle NVFP4-forward time")


def run_reference(args, cfg, d):
    M_s, N_s = REF_SAMPLE
    flops = 2.0 * M_s * N_s * cfg.K
    for _ in range(args.warmup):
        cpu_sample(d, M_s, N_s)
    times = []
    cores = 1
    t_start = time.perf_counter()
    for _ in range(args.steps):
        t, cores = cpu_sample(d, M_s, N_s)
        times.append(t)
    wall = time.perf_counter() - t_start
    fwd = statistics.median(t["fwd_nvfp4"] for t in times)
    value = flops / fwd / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (oracle, exact decoded operands)", "data": "synthetic (seeded)",
        "config": workload_config(cfg, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": cpu_sample_desc(cfg, M_s, N_s)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "ops_s": {k: statistics.median(t[k] for t in times) for k in times[0]},
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(values, world, device):
    """Element-wise max over the ranks of per-rank timings (every multi-GPU time is the
    slowest rank's); identity for one rank."""
    if world <= 1:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def workload_config(cfg, args):
    return {
        "workload": f"SquareQ W4 linear {cfg.M}x{cfg.N}x{cfg.K} (M tokens x N out x K in), rank 32, "
                    f"seed {cfg.seed}, {cfg.dist} residual" + (f", {cfg.hot_channels} hot channels"
                                                              if cfg.hot_channels else ""),
        "name": cfg.name, "M": cfg.M, "N": cfg.N, "K": cfg.K, "rank": 32,
        "codecs": ["nvfp4 (e2m1, ue4m3 block-16, fp32 global)", "int4 group-32 MSE-swept",
                   "int4 group-64 MSE-swept", "int8 per-row MSE-swept, rank-16 low-rank branch"],
        "l2": "flushed before every op, outside its events: a 256 MB write, then a read of another "
              "256 MB buffer (none of the op's inputs in L2, and no dirty lines left to write back)",
        "parallelism": f"replicas x{args.gpus}",
    }


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

class L2Flush:
    """Before every timed op: write a buffer larger than L2, then read another one, so the op
    finds none of its inputs in L2 and no dirty lines of the flush still to be written back."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.out = torch.empty((), dtype=torch.int32, device=dev)

    def __call__(self):
        import torch
        self.w.fill_(1)
        torch.amax(self.r, dim=0, out=self.out)


def time_ops(ops, flush, steps, warmup, stage_of=None):
    """Median milliseconds of each (name, fn) over `steps` runs after `warmup`, each run after an
    L2 flush, timed with CUDA events on the current stream.  stage_of[name] = [(key, stage)]
    also times those library launches with the stage events, on separate runs."""
    import torch
    import bit_quantized_frozen_b200 as sq
    stage_of = stage_of or {}
    for _ in range(warmup):
        for _, fn in ops:
            flush()
            fn()
    times = {}
    for name, fn in ops:
        keys = [k for k, _ in stage_of.get(name, [])]
        rec = {name: []} | {k: [] for k in keys}
        for it in range(steps * (2 if keys else 1)):
            inst = keys and it % 2 == 1
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            sev = {}
            if inst:
                for k, st in stage_of[name]:
                    sev[k] = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    sq.sq_set_stage_events(st, *sev[k])
            flush()
            a.record()
            fn()
            b.record()
            if inst:
                for k, st in stage_of[name]:
                    sq.sq_set_stage_events(st, None, None)
            torch.cuda.synchronize()
            if inst:
                for k in keys:
                    rec[k].append(sev[k][0].elapsed_time(sev[k][1]))
            else:
                rec[name].append(a.elapsed_time(b))
        for k, v in rec.items():
            times[k] = statistics.median(v)
    return times

def run_sq(args, cfg, d, rank, world, local_rank):
    import torch
    import bit_quantized_frozen_b200 as sq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M, N, K = cfg.M, cfg.N, cfg.K
    to_bf16 = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    R = torch.from_numpy(d["R"]).to(dev)
    x = to_bf16(d["x"])
    U = to_bf16(d["U"])
    D = to_bf16(d["D"])

    # outputs and workspaces, allocated once
    i4 = sq.Weight(sq.SQ_FMT_INT4_G32, N, K, torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                   torch.empty((N, K // 32), dtype=torch.float16, device=dev), None, U, D,
                   torch.empty((N, K // 32), dtype=torch.uint8, device=dev))
    nv = sq.Weight(sq.SQ_FMT_NVFP4, N, K, torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                   torch.empty(sq.sq_sf_bytes(N, K), dtype=torch.uint8, device=dev),
                   torch.empty(1, dtype=torch.float32, device=dev), U, D)
    i6 = sq.Weight(sq.SQ_FMT_INT4_G64, N, K, torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                   torch.empty((N, K // 64), dtype=torch.float16, device=dev), None, U, D,
                   torch.empty((N, K // 64), dtype=torch.uint8, device=dev))
    U16, D16 = U[:, :16].contiguous(), D[:, :16].contiguous()
    i8 = sq.Weight(sq.SQ_FMT_INT8_ROW, N, K, torch.empty((N, K), dtype=torch.int8, device=dev),
                   torch.empty(N, dtype=torch.float32, device=dev), None, U16, D16,
                   torch.empty(N, dtype=torch.uint8, device=dev))
    ws_i8 = sq.workspace(sq.SQ_OP_LINEAR_FWD_INT8, M, N, K, dev)
    ws_dx = sq.workspace(sq.SQ_OP_LINEAR_BWD_DX, M, N, K, dev)
    dy = torch.randn((M, N), device=dev, generator=torch.Generator(device=dev).manual_seed(cfg.seed)).to(torch.bfloat16)
    dx = torch.empty((M, K), dtype=torch.float32, device=dev)
    ws_b = sq.workspace(sq.SQ_OP_BUILD_NVFP4, 0, N, K, dev)
    ws_nv = sq.workspace(sq.SQ_OP_LINEAR_FWD_NVFP4, M, N, K, dev)
    ws_i4 = sq.workspace(sq.SQ_OP_LINEAR_FWD_INT4, M, N, K, dev)
    g_x = torch.empty(1, dtype=torch.float32, device=dev)
    y_nv = torch.empty((M, N), dtype=torch.float32, device=dev)
    y_i4 = torch.empty((M, N), dtype=torch.float32, device=dev)
    y_bf = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    W = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    Wsvd = R + U.float() @ D.float().T            # the full weight the SVD init factors (input set-up)
    omega = torch.randn((K, 32), device=dev, generator=torch.Generator(device=dev).manual_seed(cfg.seed + 1))
    up_s = torch.empty((N, 32), dtype=torch.bfloat16, device=dev)
    down_s = torch.empty((K, 32), dtype=torch.bfloat16, device=dev)
    R_s = torch.empty_like(R)
    ws_svd = sq.workspace(sq.SQ_OP_SVD_INIT, 0, N, K, dev)
    a_codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    a_sf = torch.empty(sq.sq_sf_bytes(M, K), dtype=torch.uint8, device=dev)
    a_t = torch.empty((M, 32), dtype=torch.float32, device=dev)
    ws_aq = sq.workspace(sq.SQ_OP_ACT_QUANT_NVFP4, M, 0, K, dev)
    flush = L2Flush(dev)

    ops = [
        ("build_int4", lambda: sq.sq_build_int4(R, i4.codes, i4.scales, i4.frac_idx)),
        ("build_nvfp4", lambda: sq.sq_build_nvfp4(R, nv.codes, nv.scales, nv.g_w, ws_b)),
        ("fwd_nvfp4", lambda: sq.sq_linear_fwd(nv, x, y_nv, g_x=g_x, ws=ws_nv)),
        ("fwd_nvfp4_bf16out", lambda: sq.sq_linear_fwd(nv, x, y_bf, g_x=g_x, flags=sq.SQ_OUT_BF16, ws=ws_nv)),
        ("fwd_int4", lambda: sq.sq_linear_fwd(i4, x, y_i4, ws=ws_i4)),
        ("reconstruct_nvfp4", lambda: sq.sq_reconstruct_bf16(nv, W)),
        ("reconstruct_int4", lambda: sq.sq_reconstruct_bf16(i4, W)),
        ("build_int4_g64", lambda: sq.sq_build_int4(R, i6.codes, i6.scales, i6.frac_idx, group=64)),
        ("fwd_int4_g64", lambda: sq.sq_linear_fwd(i6, x, y_i4, ws=ws_i4)),
        ("reconstruct_int4_g64", lambda: sq.sq_reconstruct_bf16(i6, W)),
        ("build_int8", lambda: sq.sq_build_int8(R, i8.codes, i8.scales, i8.frac_idx)),
        ("fwd_int8", lambda: sq.sq_linear_fwd(i8, x, y_i4, ws=ws_i8)),
        ("reconstruct_int8", lambda: sq.sq_reconstruct_bf16(i8, W)),
        ("bwd_dx_nvfp4", lambda: sq.sq_linear_bwd_dx(nv, dy, dx, ws_dx)),
        ("svd_init", lambda: sq.sq_svd_init(Wsvd, omega, SVD_ITERS, up_s, down_s, R_s, ws_svd)),
        ("act_quant_nvfp4", lambda: sq.sq_act_quant_nvfp4(x, a_codes, a_sf, g_x, lora_down=D, t=a_t, ws=ws_aq)),
        ("reconstruct_nvfp4_resid", lambda: sq.sq_reconstruct_bf16(nv, W, sq.SQ_RECON_RESIDUAL_ONLY)),
    ]
    names = [n for n, _ in ops]
    # launches timed on their own by the library's stage events (even steps; the op itself on odd
    # steps, because an event between two launches stops the second from overlapping the first)
    stages_of = {"fwd_nvfp4": [("gemm_nvfp4", sq.SQ_STAGE_GEMM)], "fwd_int4": [("gemm_int4", sq.SQ_STAGE_GEMM)],
                 "bwd_dx_nvfp4": [("gemm_bwd_dx", sq.SQ_STAGE_GEMM)],
                 "act_quant_nvfp4": [("act_pass1", sq.SQ_STAGE_ACT_PASS1), ("act_pass2", sq.SQ_STAGE_ACT_QUANT)]}
    gemm_of = {op: [k for k, _ in st] for op, st in stages_of.items()}

    # The GEMM kernel's own events are recorded on even steps only: an event between
    # the activation quantisation and the GEMM launch would stop the GEMM's set-up
    # from overlapping the quantisation, so the forward is timed on the odd steps.
    def run_step(evs, instrument_gemm=False):
        for name, fn in ops:
            flush()
            if evs is None:
                fn()
                continue
            a, b = evs[name]
            inst = instrument_gemm and name in stages_of
            if inst:
                for key, stage in stages_of[name]:
                    sq.sq_set_stage_events(stage, *evs[key])
            a.record()
            fn()
            b.record()
            if inst:
                for key, stage in stages_of[name]:
                    sq.sq_set_stage_events(stage, None, None)

    for _ in range(args.warmup):
        run_step(None)
    torch.cuda.synchronize()
    sq.sq_check_device_status(ws_nv)
    sq.sq_check_device_status(ws_i4)
    sq.sq_check_device_status(ws_i8)

    stage_keys = [k for v in gemm_of.values() for k in v]
    keys = names + stage_keys
    evs = [{k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for k in keys}
           for _ in range(args.steps)]
    outer = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    sampler = None
    if rank == 0 and not args.no_clocks:
        sampler = ClockSampler(physical_gpu_index(local_rank))
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    outer[0].record()
    for s in range(args.steps):
        run_step(evs[s], instrument_gemm=(s % 2 == 0))
    outer[1].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    sq.sq_check_device_status(ws_nv)
    sq.sq_check_device_status(ws_i4)

    even = evs[0::2]
    odd = evs[1::2] or evs                     # a single step: the op carries the stage events
    per_op = {k: statistics.median(e[k][0].elapsed_time(e[k][1])
                                   for e in (even if k in stage_keys else odd if k in gemm_of else evs))
              for k in keys}   # ms, median over the steps
    outer_ms = outer[0].elapsed_time(outer[1]) / max(args.steps, 1)
    vals = max_over_ranks([per_op[k] for k in keys] + [outer_ms], world, dev)
    per_op = dict(zip(keys, vals[:-1]))
    outer_ms = vals[-1]

    # end to end through the C ABI with host buffers: H2D of x, forward, D2H of y.
    # Steps are independent, so step i+1's upload and forward run on one stream while
    # step i's download runs on another (opposite directions of the link); device x and
    # y are double buffered.  Every step still carries both copies in full.
    e2e = None
    if not args.no_e2e:
        x_host = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
        y_host = torch.empty((M, N), dtype=torch.float32).pin_memory()
        x_dev = [torch.empty_like(x), torch.empty_like(x)]
        y_dev = [y_nv, torch.empty_like(y_nv)]
        s_main = torch.cuda.current_stream()
        s_d2h = torch.cuda.Stream()
        fwd_done = [torch.cuda.Event(), torch.cuda.Event()]
        d2h_done = [torch.cuda.Event(), torch.cuda.Event()]

        def e2e_step(i):
            b = i % 2
            s_main.wait_event(d2h_done[b])                # y_dev[b] was downloaded (step i - 2)
            x_dev[b].copy_(x_host, non_blocking=True)
            sq.sq_linear_fwd(nv, x_dev[b], y_dev[b], g_x=g_x, ws=ws_nv)
            fwd_done[b].record(s_main)
            s_d2h.wait_event(fwd_done[b])
            with torch.cuda.stream(s_d2h):
                y_host.copy_(y_dev[b], non_blocking=True)
            d2h_done[b].record(s_d2h)

        for b in range(2):                                # the events exist before the first wait
            d2h_done[b].record(s_d2h)
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        reps = 6
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_main)
        for i in range(reps):
            e2e_step(i)
        s_main.wait_stream(s_d2h)
        e1.record(s_main)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / reps], world, dev)[0]
        e2e = {"value": world * 2.0 * M * N * K / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(M * K * 2), "d2h_bytes_per_step": int(M * N * 4),
               "ms_per_step": e2e_ms,
               "path": "pinned x -> device, sq_linear_fwd (NVFP4), y -> pinned host; step i+1's upload "
                       "and forward overlap step i's download (two streams, double-buffered x and y)"}
    return per_op, outer_ms, clocks, e2e


def rate_entries(per_op, M, N, K, peaks, peak_src):
    """{op: {ms, rate, frac of its roofline, alu (the ALU-bound kernels)}} for median times."""
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    work = op_work(M, N, K)
    ops = {}
    for k, ms in per_op.items():
        unit, amount = work[k]
        rate = amount / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
        if unit == "GB/s":
            frac, peak = rate / peaks["hbm_gbs"], "hbm"
        elif k == "svd_init":
            frac, peak = rate / FP32_ALU_TFLOPS, "fp32 FMA issue"
        else:
            fp4 = k in ("fwd_nvfp4", "fwd_nvfp4_bf16out", "gemm_nvfp4")   # the backward's GEMM runs in bf16
            peak_v = fp4_peak if fp4 else peaks["bf16_tflops"]
            frac, peak = rate / peak_v, "fp4 tensor" if fp4 else "bf16 tensor"
        src = "148 SMs x 128 lanes x 2 flop x 1.965 GHz" if k == "svd_init" else peak_src
        ops[k] = {"ms": ms, unit: rate, "frac": frac, "of": f"{peak} ({src})"}
        if k in ALU_OPS:
            gops = ALU_OPS[k] * N * K / (ms * 1e-3) / 1e9
            ops[k]["alu"] = {"Gop/s": gops, "frac": gops / ALU_GOPS, "ops_per_element": ALU_OPS[k],
                             "of": "fp32 lane-op issue, 148 SMs x 128 lanes x 1.965 GHz (unit counts, max clock)"}
    return ops


def summarise(args, cfg, per_op, outer_ms, clocks, e2e, world, cpu, extra=None):
    peaks, peak_src = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    M, N, K = cfg.M, cfg.N, cfg.K
    ops = rate_entries(per_op, M, N, K, peaks, peak_src)
    fwd_tflops = 2.0 * M * N * K / (per_op["fwd_nvfp4"] * 1e-3) / 1e12
    gemm_tflops = 2.0 * M * N * K / (per_op["gemm_nvfp4"] * 1e-3) / 1e12
    traffic, traffic_src = profiled_traffic(cfg.name)
    step_ms = sum(per_op[k] for k in LAUNCHES_PER_STEP)
    base = PAGES_FP4_TFLOPS.get(cfg.name)
    line = {
        "metric": METRIC,
        "value": world * fwd_tflops,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": (world * fwd_tflops / base) if base else None,
        "vs_baseline_note": ("pages' RTX 5080 (sm_120) cuBLASLt fp4 GEMM-only time for this shape; "
                             "context, not a target") if base else None,
        "dtype": "e2m1 x e2m1 with ue4m3 block-16 scales -> fp32 (NVFP4 headline); bf16 x bf16 -> fp32 (int4 path)",
        "data": "synthetic (seeded numpy; shapes/distributions of the pages' model layers)",
        "config": workload_config(cfg, args),
        "roofline": {
            "kernel": "sq_gemm_kernel<NVFP4> (tcgen05 block-scaled GEMM + low-rank step + epilogue)",
            "bound": "tensor",
            "achieved": gemm_tflops,
            "peak": fp4_peak,
            "unit": "TFLOP/s",
            "frac": gemm_tflops / fp4_peak,
            "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {FP4_PER_BF16} (nominal fp4/bf16)",
            "traffic": traffic,
            "traffic_source": traffic_src,
            "algorithmic": f"2*M*N*K = {2.0 * M * N * K:.4g} flop per launch",
        },
        "ops": ops,
        "ms_per_step_with_flushes": outer_ms,
        "gpu_launches": sum(LAUNCHES_PER_STEP.values()) * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if extra:
        for name, times in extra.get("per_config", {}).items():
            c = si.CONFIGS[name]
            line.setdefault("per_config", {})[name] = {
                "M": c.M, "N": c.N, "K": c.K, "ops": rate_entries(times, c.M, c.N, c.K, peaks, peak_src)}
        if "stack" in extra:
            line["builder_stack"] = extra["stack"]
    return line


PER_CONFIG = ["tiny_64x256x512", "proj_1536x3072x3072", "qkv_1536x9216x3072", "large_4480x6144x6144",
              "down_4480x6144x16384"]


def run_configs(headline, dev):
    """The forward, activation quantiser, builders and reconstructs on every other configuration,
    5 timed runs each (median) after 2 warm-up runs, L2 flushed before each."""
    import torch
    import bit_quantized_frozen_b200 as sq
    flush = L2Flush(dev)
    out = {}
    for name in PER_CONFIG:
        if name == headline:
            continue
        cfg = si.CONFIGS[name]
        d = si.make_config(name)
        M, N, K = cfg.M, cfg.N, cfg.K
        to_bf16 = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        R, x, U, D = torch.from_numpy(d["R"]).to(dev), to_bf16(d["x"]), to_bf16(d["U"]), to_bf16(d["D"])
        nv = sq.Weight(sq.SQ_FMT_NVFP4, N, K, torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                       torch.empty(sq.sq_sf_bytes(N, K), dtype=torch.uint8, device=dev),
                       torch.empty(1, dtype=torch.float32, device=dev), U, D)
        i4 = sq.Weight(sq.SQ_FMT_INT4_G32, N, K, torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                       torch.empty((N, K // 32), dtype=torch.float16, device=dev), None, U, D,
                       torch.empty((N, K // 32), dtype=torch.uint8, device=dev))
        ws_b = sq.workspace(sq.SQ_OP_BUILD_NVFP4, 0, N, K, dev)
        ws_nv = sq.workspace(sq.SQ_OP_LINEAR_FWD_NVFP4, M, N, K, dev)
        ws_i4 = sq.workspace(sq.SQ_OP_LINEAR_FWD_INT4, M, N, K, dev)
        ws_aq = sq.workspace(sq.SQ_OP_ACT_QUANT_NVFP4, M, 0, K, dev)
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
        W = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        g_x = torch.empty(1, dtype=torch.float32, device=dev)
        a_codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        a_sf = torch.empty(sq.sq_sf_bytes(M, K), dtype=torch.uint8, device=dev)
        a_t = torch.empty((M, 32), dtype=torch.float32, device=dev)
        ops = [
            ("build_nvfp4", lambda: sq.sq_build_nvfp4(R, nv.codes, nv.scales, nv.g_w, ws_b)),
            ("build_int4", lambda: sq.sq_build_int4(R, i4.codes, i4.scales, i4.frac_idx)),
            ("act_quant_nvfp4", lambda: sq.sq_act_quant_nvfp4(x, a_codes, a_sf, g_x, lora_down=D, t=a_t, ws=ws_aq)),
            ("fwd_nvfp4", lambda: sq.sq_linear_fwd(nv, x, y, g_x=g_x, ws=ws_nv)),
            ("fwd_int4", lambda: sq.sq_linear_fwd(i4, x, y, ws=ws_i4)),
            ("reconstruct_nvfp4", lambda: sq.sq_reconstruct_bf16(nv, W)),
            ("reconstruct_nvfp4_resid", lambda: sq.sq_reconstruct_bf16(nv, W, sq.SQ_RECON_RESIDUAL_ONLY)),
        ]
        stage_of = {"fwd_nvfp4": [("gemm_nvfp4", sq.SQ_STAGE_GEMM)],
                    "act_quant_nvfp4": [("act_pass1", sq.SQ_STAGE_ACT_PASS1), ("act_pass2", sq.SQ_STAGE_ACT_QUANT)]}
        out[name] = time_ops(ops, flush, steps=5, warmup=2, stage_of=stage_of)
        sq.sq_check_device_status(ws_nv)
        del R, x, U, D, nv, i4, ws_b, ws_nv, ws_i4, ws_aq, y, W, a_codes, a_sf, a_t, ops
        torch.cuda.empty_cache()
    return out


def run_stack(dev, count=si.STACK_COUNT):
    """The down-projection shape's builder stack: `count` residual weights [6144, 16384] fp32 drawn
    one after another into one device buffer (untimed), each built by the three builders (timed,
    L2 flushed before each build)."""
    import torch
    import bit_quantized_frozen_b200 as sq
    N, K = 6144, 16384
    flush = L2Flush(dev)
    Rb = torch.empty((N, K), dtype=torch.float32, device=dev)
    c4 = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    s4 = torch.empty((N, K // 32), dtype=torch.float16, device=dev)
    f4 = torch.empty((N, K // 32), dtype=torch.uint8, device=dev)
    cn = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sn = torch.empty(sq.sq_sf_bytes(N, K), dtype=torch.uint8, device=dev)
    gn = torch.empty(1, dtype=torch.float32, device=dev)
    ws_b = sq.workspace(sq.SQ_OP_BUILD_NVFP4, 0, N, K, dev)
    c8 = torch.empty((N, K), dtype=torch.int8, device=dev)
    s8 = torch.empty(N, dtype=torch.float32, device=dev)
    f8 = torch.empty(N, dtype=torch.uint8, device=dev)
    builders = [("build_int4", lambda: sq.sq_build_int4(Rb, c4, s4, f4), 4 + 0.5 + 2 / 32 + 1 / 32),
                ("build_nvfp4", lambda: sq.sq_build_nvfp4(Rb, cn, sn, gn, ws_b), 4 + 0.5 + 1 / 16),
                ("build_int8", lambda: sq.sq_build_int8(Rb, c8, s8, f8), 4 + 1)]
    ev = {b: [] for b, _, _ in builders}
    for i in range(count):
        si.make_stack_residual_device(i, Rb, N, K)
        for b, fn, _ in builders:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush()
            e0.record()
            fn()
            e1.record()
            ev[b].append((e0, e1))
    torch.cuda.synchronize()
    res = {"weights": count, "shape": [N, K],
           "inputs": "seeded Student-t(4) residuals (std 1/sqrt(K)), drawn on the device per weight into "
                     "one buffer, untimed; L2 flushed before each build"}
    for b, _, bpe in builders:
        ms = [a.elapsed_time(e) for a, e in ev[b]]
        tot = sum(ms)
        res[b] = {"total_ms": tot, "ms_per_weight_median": statistics.median(ms),
                  "GB/s": count * N * K * bpe / (tot * 1e-3) / 1e9}
    del Rb, c4, s4, f4, cn, sn, gn, ws_b, c8, s8, f8
    torch.cuda.empty_cache()
    return res


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = si.CONFIGS[args.config]
    if args.impl == "reference":
        if rank != 0:
            return
        d = si.make_config(cfg.name)
        run_reference(args, cfg, d)
        return
    import torch
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    d = si.make_config(cfg.name)
    per_op, outer_ms, clocks, e2e = run_sq(args, cfg, d, rank, world, local_rank)
    extra = None
    if rank == 0 and world == 1 and not args.no_extra:
        dev = torch.device("cuda", local_rank)
        extra = {"per_config": run_configs(cfg.name, dev), "stack": run_stack(dev)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        M_s, N_s = CPU_SAMPLE
        t, cores = cpu_sample(d, M_s, N_s)
        cpu = {"value": 2.0 * M_s * N_s * cfg.K / t["fwd_nvfp4"] / 1e12, "unit": "TFLOP/s", "cores": cores,
               "kind": "oracle", "sample": cpu_sample_desc(cfg, M_s, N_s), "ops_s": t}
    if rank == 0:
        print(json.dumps(summarise(args, cfg, per_op, outer_ms, clocks, e2e, world, cpu, extra)), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
