"""Host-side pieces of bench.py that need no GPU: the algorithmic byte count
per vector and the clock / throttle-reason summary of the sampled
nvidia-smi lines."""

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_bytes_per_vector():
    b = load_bench()
    # 2d bytes of fp16 in, d/2 bytes of nibbles and 4 bytes per group out
    assert b.fwd_bytes(64, 64) == 128 + 32 + 4 == 164
    assert b.fwd_bytes(128, 32) == 256 + 64 + 16 == 336
    assert b.fwd_bytes(256, 256) == 512 + 128 + 4
    # one launch over the 6,291,456-vector SmolLM2-1.7B-shaped cache
    assert 6291456 * b.fwd_bytes(64, 64) == 1031798784


def sample(sm, mx, hw="Not Active", thermal="Not Active", sw_thermal="Not Active",
           power="Not Active"):
    return f"0, {sm}, {mx}, 600.5, 0x0, {hw}, {thermal}, {sw_thermal}, {power}"


def test_clock_summary_median_min_and_reasons():
    b = load_bench()
    c = b.ClockSampler(0)
    c.lines = [(1.0, sample(1965, 1965)), (2.0, sample(1900, 1965, power="Active")),
               (3.0, sample(1700, 1965)), (4.0, "garbage line"), (5.0, sample(1965, 1965))]
    s = c.summary()
    assert s["samples"] == 4
    assert s["sm_mhz"] == 1932.5 and s["sm_min_mhz"] == 1700 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_keeps_the_marked_window():
    b = load_bench()
    c = b.ClockSampler(0)
    c.lines = [(1.0, sample(800, 1965, thermal="Active")), (10.0, sample(1965, 1965)),
               (10.5, sample(1955, 1965)), (20.0, sample(900, 1965, hw="Active"))]
    c.marks = [9.9, 10.6]
    s = c.summary()
    assert s["samples"] == 2 and s["sm_min_mhz"] == 1955 and s["reasons"] == []


def test_clock_summary_without_samples():
    b = load_bench()
    s = b.ClockSampler(0).summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["reasons"] == []


def test_sweep_cells_and_bytes_per_step():
    b = load_bench()
    cells = b.sweep_cells()
    assert len(cells) == 12  # 3 d x 2 groups x 2 rotations, each forward then inverse
    assert (256, 256, 0) in cells and (64, 32, 1) in cells
    n = 8388608
    per_step = b.sweep_fp16_bytes_per_step({64: n, 128: n, 256: n})
    # every (d, g, rot) cell moves n*d*2 bytes of fp16 in the forward and out
    # of the inverse launch
    assert per_step == 4 * 2 * n * (64 + 128 + 256) * 2


def test_cell_record_fraction_of_peak():
    b = load_bench()
    n = 8388608
    algo = n * b.fwd_bytes(256, 256)
    ms = [algo / 4000e9 * 1e3, algo / 3000e9 * 1e3, algo / 5000e9 * 1e3]
    r = b.cell_record(256, 256, 0, "fwd", ms, n, 6543.4)
    assert r["cell"] == "kvq_fwd_kernel d=256 g=256 srft"
    assert abs(r["algo_gbs_median"] - 4000) < 1e-6
    assert abs(r["frac_median"] - 4000 / 6543.4) < 1e-9
    assert abs(r["frac_best"] - 5000 / 6543.4) < 1e-9


class FakeNvml:
    NVML_CLOCK_SM = 1

    def __init__(self, seq):
        self.seq = list(seq)

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, which):
        return self.seq[0][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.seq.pop(0)[1] if len(self.seq) > 1 else self.seq[0][1]


def test_nvml_sampler_reads_clock_and_reason_bits():
    b = load_bench()
    s = b.NvmlSampler(None, FakeNvml([(1965, 0x0)]))
    assert s.max_mhz == 1965
    s.samples = [(1.0, 1965.0, set()), (2.0, 1800.0, {"sw_power_cap"}),
                 (3.0, 1500.0, {"hw_slowdown"}), (4.0, 1900.0, set())]
    s.marks = [1.5, 3.5]
    out = s.summary()
    assert out["samples"] == 2 and out["sm_mhz"] == 1650.0 and out["sm_min_mhz"] == 1500.0
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"] and out["source"] == "nvml 10 ms"
    # the reason bits NVML reports (clock-event reasons)
    assert b.NvmlSampler.BITS == {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
                                  "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}


def test_nvml_sampler_thread_collects_samples():
    import time as _t
    b = load_bench()
    s = b.NvmlSampler(None, FakeNvml([(1965, 0x4)]), period=0.002)
    s.start()
    s.mark()
    _t.sleep(0.05)
    s.mark()
    s.stop()
    out = s.summary()
    assert out["samples"] >= 3 and out["reasons"] == ["sw_power_cap"]


def test_relaunch_under_torchrun(monkeypatch):
    b = load_bench()
    cmd = b.relaunch_command(["--gpus", "4", "--steps", "2"], 4, 29500)
    i = cmd.index("torch.distributed.run")
    assert cmd[i - 1] == "-m" and "--nproc-per-node" in cmd
    assert cmd[cmd.index("--nproc-per-node") + 1] == "4"
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "2"] and cmd[-5].endswith("bench.py")

    class A:
        gpus, impl = 2, "kvq"
    monkeypatch.setenv("WORLD_SIZE", "4")
    import pytest
    with pytest.raises(SystemExit, match="WORLD_SIZE=4"):
        b.maybe_relaunch(A, [])
    monkeypatch.delenv("WORLD_SIZE")
    monkeypatch.setattr(b.torch.cuda, "is_available", lambda: False)
    with pytest.raises(SystemExit, match="0 CUDA device"):
        b.maybe_relaunch(A, [])
