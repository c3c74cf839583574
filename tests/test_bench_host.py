"""Host-side pieces of bench.py, on the CPU: the clock record it attaches to the JSON line, the
physical GPU index the sampler queries, and the rule that the roofline's DRAM traffic is taken
from the committed ncu summary only while the GEMM source is the one that was profiled."""
import bench


class FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def sampled(lines):
    s = bench.ClockSampler(0)
    s.proc = FakeProc()
    s.lines = list(lines)
    return s.stop()


def line(sm, smax=1965, hw="Not Active", hwt="Not Active", swt="Not Active", cap="Not Active", util=100):
    return f"{sm}, {smax}, 812.5, {hw}, {hwt}, {swt}, {cap}, {util}"


def test_clocks_median_under_load_and_reasons():
    rec = sampled([line(1200, util=0), line(1965), line(1950), line(1800, cap="Active"), line(900, util=0),
                   "garbage", "", "[N/A], 1965, 0, Not Active, Not Active, Not Active, Not Active, 100"])
    assert rec["sm_mhz"] == 1950.0                 # median of the three samples under load
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples"] == 5 and rec["samples_under_load"] == 3


def test_clocks_reasons_only_count_under_load():
    rec = sampled([line(1965), line(1965, hw="Active", util=0), line(1965, hwt="Active", swt="Active")])
    assert rec["reasons"] == ["hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clocks_idle_run_uses_every_sample():
    rec = sampled([line(1100, util=0), line(1300, util=0)])
    assert rec["sm_mhz"] == 1200.0 and rec["samples_under_load"] == 0


def test_clocks_without_samples():
    assert sampled([])["samples"] == 0
    s = bench.ClockSampler(0)                      # never started (no nvidia-smi)
    assert s.stop() is None


def test_physical_gpu_index(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "5, 2")
    assert bench.physical_gpu_index(0) == 5 and bench.physical_gpu_index(1) == 2
    assert bench.physical_gpu_index(3) == 3        # beyond the list: the local rank
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-1a2b")
    assert bench.physical_gpu_index(0) == 0        # a UUID: the local rank
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.physical_gpu_index(1) == 1


def test_traffic_only_for_the_profiled_source(monkeypatch):
    value, src = bench.profiled_traffic(bench.HEADLINE)
    assert src == "ncu" and value > 0              # the committed summary matches the source
    assert bench.profiled_traffic("no_such_workload") == (None, "no capture for this workload")
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic(bench.HEADLINE) == (None, "kernel changed since the ncu capture")


def test_traffic_hash_ignores_comments_only():
    src = {rel: open(f"{bench.ROOT}/{rel}").read() for rel in bench.GEMM_SOURCES}
    base = bench.gemm_source_hash(src.__getitem__)
    assert base == bench.gemm_source_hash()
    first = bench.GEMM_SOURCES[0]
    commented = dict(src, **{first: "// a new comment\n/* and a\n   block */\n" + src[first] + "\n\n// tail\n"})
    assert bench.gemm_source_hash(commented.__getitem__) == base
    edited = dict(src, **{first: src[first].replace("kStages", "kStages ", 1) + "\nstatic int extra;\n"})
    assert bench.gemm_source_hash(edited.__getitem__) != base
