"""Host-side pieces of the benchmark that need no GPU: the clock record parsed
from nvidia-smi's CSV stream, and the DRAM-traffic lookup that is valid only
for the kernel sources it was captured from."""
import json
import os

import bench


class _FakeProc:
    def __init__(self, out):
        self._out = out

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self._out, ""

    def kill(self):
        pass


def _sampler(first, rest):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.proc = _FakeProc(rest)
    s.first = first
    s.path = None
    return s


# fields: clocks.sm, clocks.max.sm, power.draw, active reasons, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
IDLE = "345, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
LOAD = "1965, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
CAPPED = "1750, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active\n"


def test_clock_median_under_load_and_reasons():
    rec = _sampler(IDLE, LOAD * 4 + CAPPED * 3).stop()
    # the idle first sample draws under half the peak power: not "under load"
    assert rec["samples"] == 8 and rec["samples_under_load"] == 7
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert "note" not in rec


def test_clock_first_sample_alone_is_reported_with_a_note():
    rec = _sampler(LOAD, "").stop()
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1965.0
    assert "note" in rec


def test_clock_no_sampler():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.proc = None
    assert s.stop() is None


def test_traffic_lookup_follows_the_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    # a tree of its own: the hash covers its (here empty) kernel sources
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    good = {"csrc_hash": bench.csrc_hash(), "workloads": {"w": {"fwd": {"dram_bytes": 123.0}}}}
    (prof / "traffic.json").write_text(json.dumps(good))
    assert bench.measured_traffic("w", "fwd") == 123.0
    assert bench.measured_traffic("w", "dx") is None
    stale = dict(good, csrc_hash="0" * 16)
    (prof / "traffic.json").write_text(json.dumps(stale))
    assert bench.measured_traffic("w", "fwd") is None
    os.remove(prof / "traffic.json")
    assert bench.measured_traffic("w", "fwd") is None


def test_end_to_end_copies_only_the_steps_results():
    # a two-layer block: y of the last layer, dx of the first, every layer's dcoef / dw_base
    assert bench.result_keys(0, 2, "fwdbwd") == ["dx", "dcoef", "dwb"]
    assert bench.result_keys(1, 2, "fwdbwd") == ["y", "dcoef", "dwb"]
    assert bench.result_keys(0, 1, "fwdbwd") == ["y", "dx", "dcoef", "dwb"]
    assert bench.result_keys(0, 1, "fwd") == ["y"]
    assert bench.result_keys(0, 2, "fwd") == []
