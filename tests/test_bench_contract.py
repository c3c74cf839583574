"""The bench's JSON line, checked on the host (no GPU): every op the step times has its
algorithmic work and launch count, and summarise() emits the keys and units the line must carry
(metric, value, unit, roofline with bound/achieved/peak/frac/traffic, e2e, cpu_baseline, clocks,
gpu_launches) with values consistent with the timings fed in."""
import argparse
import ast
import json
import os

import bench
import synth_inputs as si

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def step_op_names():
    """The op names of run_sq's step list, read from bench.py's source."""
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    for node in ast.walk(tree):
        if isinstance(node, ast.FunctionDef) and node.name == "run_sq":
            for sub in ast.walk(node):
                if isinstance(sub, ast.Assign) and any(getattr(t, "id", None) == "ops" for t in sub.targets):
                    return [elt.elts[0].value for elt in sub.value.elts]
    raise AssertionError("run_sq's op list not found")


def test_every_step_op_has_work_and_launch_count():
    names = step_op_names()
    work = bench.op_work(4480, 16384, 6144)
    assert sorted(names) == sorted(bench.LAUNCHES_PER_STEP)
    for n in names:
        assert n in work, n
    for g in ("gemm_nvfp4", "gemm_int4", "gemm_bwd_dx"):
        assert g in work


def test_summarise_line():
    cfg = si.CONFIGS[bench.HEADLINE]
    args = argparse.Namespace(gpus=1, steps=10, warmup=3)
    work = bench.op_work(cfg.M, cfg.N, cfg.K)
    per_op = {k: 0.5 for k in work}                               # ms
    per_op["gemm_nvfp4"] = 0.25
    per_op["fwd_nvfp4"] = 0.30
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5}
    e2e = {"value": 150.0, "unit": "TFLOP/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 2}
    cpu = {"value": 0.04, "unit": "TFLOP/s", "cores": 16, "kind": "oracle", "sample": "s"}
    line = bench.summarise(args, cfg, per_op, 8.0, clocks, e2e, 1, cpu)
    json.dumps(line)                                               # serialisable
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "ops", "gpu_launches",
              "clocks", "e2e", "cpu_baseline"):
        assert k in line, k
    flops = 2.0 * cfg.M * cfg.N * cfg.K
    assert abs(line["value"] - flops / 0.30e-3 / 1e12) < 1e-6 * line["value"]
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True and line["scaling"] == "weak"
    rf = line["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s"
    assert abs(rf["achieved"] - flops / 0.25e-3 / 1e12) < 1e-6 * rf["achieved"]
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-12
    assert line["gpu_launches"] == sum(bench.LAUNCHES_PER_STEP.values()) * args.steps
    assert line["ms_per_step"] == sum(per_op[k] for k in bench.LAUNCHES_PER_STEP)
    assert line["config"]["workload"].startswith("SquareQ W4 linear 4480x16384x6144")
    for k, v in line["ops"].items():
        assert v["ms"] == per_op[k] and "frac" in v and "of" in v
    assert line["ops"]["svd_init"]["of"].startswith("fp32 FMA issue")
    assert line["ops"]["fwd_nvfp4_bf16out"]["of"].startswith("fp4 tensor")
