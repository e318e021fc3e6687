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
