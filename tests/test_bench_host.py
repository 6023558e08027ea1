"""Host-side logic of bench.py that decides what its JSON line reports (no
GPU): the clock summary over the timed region, the traffic record keyed by
the kernel sources, and the whole-job throughput."""

import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sampler(samples, window):
    """A ClockSampler holding recorded nvidia-smi lines, without starting it."""
    c = bench.ClockSampler(0)
    c.lines = [(t, ln) for t, ln in samples]
    c.window = window
    return c


IDLE = "1965, 1965, Not Active, Not Active, Not Active, Not Active"
CAPPED = "1860, 1965, Not Active, Not Active, Not Active, Active"
THERMAL = "1500, 1965, Not Active, Active, Not Active, Not Active"


def test_clock_summary_takes_the_samples_inside_the_region():
    samples = [(0.95, THERMAL), (1.00, IDLE), (1.05, CAPPED), (1.10, IDLE), (1.30, THERMAL)]
    s = _sampler(samples, (0.99, 1.12)).summary()
    assert s["samples_in_region"] == 3
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    # a reason active in any sample inside the region is reported; the
    # thermal samples outside it are not
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_of_a_region_shorter_than_the_sampling_period():
    """No sample falls inside: the first one after the region stands in for
    it, and samples_in_region says 0."""
    samples = [(0.90, CAPPED), (1.20, THERMAL), (1.40, IDLE)]
    s = _sampler(samples, (1.00, 1.01)).summary()
    assert s["samples_in_region"] == 0
    assert s["sm_mhz"] == 1500.0
    assert s["reasons"] == ["hw_thermal_slowdown"]


def test_clock_summary_skips_malformed_lines_and_handles_none():
    samples = [(1.0, "[N/A], 1965, Not Active, Not Active, Not Active, Not Active"), (1.1, "garbage"),
               (1.2, CAPPED)]
    s = _sampler(samples, (0.5, 1.5)).summary()
    assert s["sm_mhz"] == 1860.0 and s["reasons"] == ["sw_power_cap"]
    empty = _sampler([], (0.0, 1.0)).summary()
    assert empty == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples_in_region": 0}


def test_traffic_record_is_used_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    rec = {"digest": bench.kernel_digest(), "bytes_per_step": {"split-quant": 123, "gemm": 45}}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(p))
    assert bench.measured_traffic("split-quant") == 123
    assert bench.measured_traffic("gemm") == 45
    assert bench.measured_traffic("other") is None
    # another digest: the kernels changed since the counters were taken
    rec["digest"] = "0" * 16
    p.write_text(json.dumps(rec))
    assert bench.measured_traffic("split-quant") is None
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(tmp_path / "missing.json"))
    assert bench.measured_traffic("split-quant") is None


def test_kernel_digest_follows_every_listed_source(tmp_path, monkeypatch):
    """Changing any byte of any listed kernel source changes the digest."""
    csrc = tmp_path / "quantized_gemm_column_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.KERNEL_SOURCES:
        (csrc / f).write_bytes(b"x")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d0 = bench.kernel_digest()
    for f in bench.KERNEL_SOURCES:
        (csrc / f).write_bytes(b"y")
        assert bench.kernel_digest() != d0, f
        (csrc / f).write_bytes(b"x")
    assert bench.kernel_digest() == d0


def test_committed_traffic_record_names_both_groups():
    with open(os.path.join(ROOT, "profiles", "traffic_qkv_step.json")) as fh:
        rec = json.load(fh)
    assert len(rec["digest"]) == 16
    assert set(rec["bytes_per_step"]) == {"split-quant", "gemm"}
    assert all(isinstance(v, int) and v > 0 for v in rec["bytes_per_step"].values())


@pytest.mark.parametrize("world", [1, 2, 8])
def test_job_value_is_the_whole_job_rate(world):
    # one step of 2 * (2 l m n) FLOPs at the QKV shape in 0.1 ms per rank
    v = bench.job_value(bench.FLOPS_PER_STEP, world, 0.1)
    assert v == pytest.approx(world * bench.FLOPS_PER_STEP / 1e-4 / 1e12)
    assert bench.FLOPS_PER_STEP == 4 * 8192 * 1024 * 4096
