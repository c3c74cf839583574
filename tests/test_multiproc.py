"""The N > 1 host paths of bench.py on CPU: ranks as processes over gloo.

The layer has no exchange step (replicas only), so what more than one rank adds
is host logic: every device time is the maximum over ranks, and the reference
arm (the CPU oracle) runs and prints on rank 0 alone.
"""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, store_path, out):
    # a file rendezvous: no TCP port to race for
    dist.init_process_group("gloo", init_method=f"file://{store_path}", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench
        vals = bench.max_over_ranks([float(rank), 10.0 - rank, 5.0, 0.5 * rank], world, "cpu")
        out[rank] = vals
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks(tmp_path):
    with mp.get_context("spawn").Manager() as mgr:       # no fork of a multi-threaded process
        out = mgr.dict()
        mp.spawn(_rank_main, args=(2, str(tmp_path / "store"), out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1] == [1.0, 10.0, 5.0, 0.5]


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 1.0], 1, "cpu") == [3.0, 1.0]


def test_reference_arm_under_torchrun_two_ranks():
    # --standalone binds the rendezvous store to a port of its own choosing: no window between
    # picking a free port here and torchrun binding it
    cmd = [sys.executable, "-m", "torch.distributed.run", "--standalone", "--local-addr", "127.0.0.1",
           "--nproc-per-node", "2", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "tiny_64x256x512"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
