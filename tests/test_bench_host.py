"""Host-side pieces of bench.py (no GPU): the per-stage timing proxy, the
traffic lookup guard and the clock-sample summary."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _FakeEvent:
    clock = 0.0

    def __init__(self, enable_timing=False, external=False):
        self.t = None

    def record(self, stream=None):
        _FakeEvent.clock += 1.0
        self.t = _FakeEvent.clock

    def elapsed_time(self, end):
        return end.t - self.t  # "milliseconds"


class _FakeTorch:
    class cuda:
        Event = _FakeEvent


class _FakeMsa:
    GATHER_DEVICE_PULL = 1

    def __init__(self):
        self.calls = []

    def route(self, *a, **k):
        self.calls.append("route")
        _FakeEvent.clock += 4.0  # the call "takes" 4 ticks between its events

    def gather(self, *a, **k):
        self.calls.append("gather")

    def attend(self, *a, **k):
        self.calls.append("attend")
        _FakeEvent.clock += 1.0

    def sync_check(self):
        self.calls.append("sync_check")


def test_stage_clock_brackets_each_stage_call():
    msa = _FakeMsa()
    clock = bench.StageClock(msa, _FakeTorch)
    for _ in range(2):  # two layers
        clock.route(1, 2, k=3)
        clock.gather()
        clock.attend()
    clock.sync_check()  # not a stage: passed through untimed
    assert msa.calls == ["route", "gather", "attend"] * 2 + ["sync_check"]
    assert clock.GATHER_DEVICE_PULL == 1  # constants pass through
    assert [m[0] for m in clock.marks] == ["route", "gather", "attend"] * 2
    us = clock.per_call_us(2)
    # end - start = 1 tick for the end event's own record + the call's ticks; 1 tick = 1 ms = 1000 us
    assert us == {"route": 5000.0, "gather": 1000.0, "attend": 2000.0}


def test_traffic_lookup_needs_the_current_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()[:16]
    (prof / "traffic.json").write_text(json.dumps(
        {"k_kernel": {"10m": {"bytes_per_launch": 123.0, "source_sha": sha}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("k_kernel", "k.cu", "10m") == 123.0
    assert bench.traffic_for("k_kernel", "k.cu", "10m", bytes_scale=2.0) == 246.0
    assert bench.traffic_for("k_kernel", "k.cu", "1m") is None
    assert bench.traffic_for("other_kernel", "k.cu", "10m") is None
    src.write_text("kernel v2\n")  # the kernel changed since the counters were taken
    assert bench.traffic_for("k_kernel", "k.cu", "10m") is None


def test_committed_traffic_matches_the_committed_kernels():
    """Every committed DRAM-traffic entry was taken on (or is marked as
    unchanged from) the kernel source now in the tree."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    files = {"score_tc_kernel": "score_tc.cu", "score_pf_kernel": "score_pf.cu"}
    for kernel, entries in d.items():
        path = os.path.join(ROOT, "routed_sparse_attention_msa_b200", "csrc", files[kernel])
        sha = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
        for workload, e in entries.items():
            assert e["source_sha"] == sha, (kernel, workload)
            assert e["bytes_per_launch"] > 0


@pytest.mark.parametrize("lines, reasons", [
    (["1965, 1965, 800.1, Not Active, Not Active, Not Active, Not Active"] * 3, []),
    (["1342, 1965, 990.0, Not Active, Not Active, Not Active, Active",
      "1350, 1965, 995.0, Not Active, Not Active, Not Active, Active"], ["sw_power_cap"]),
    (["1000, 1965, 700.0, Active, Not Active, Not Active, Not Active",
      "garbage line", "[N/A], 1965, 0, Not Active, Not Active, Not Active, Not Active"], ["hw_slowdown"]),
])
def test_clock_summary(lines, reasons):
    c = bench.ClockSampler("GPU-x")
    c.lines = lines
    s = c.summary()
    assert s["reasons"] == reasons
    assert s["sm_max_mhz"] == 1965.0
    assert s["samples"] == sum(1 for ln in lines if ln[0].isdigit())
