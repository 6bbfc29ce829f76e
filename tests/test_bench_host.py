"""bench.py's host-side helpers on the CPU: the NVML clock sampler (against a fake NVML
module: it only reads), the one re-measurement of a timed region that saw a hardware or
thermal slowdown, the hash guard that reports ncu traffic only for the kernel source it
was captured on, the peak-file fallback and the whole-job value."""
import os
import shutil
import sys
import time
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_nvml(clock_seq, reason_bits):
    nv = types.SimpleNamespace()
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    nv.nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80
    it = iter(clock_seq)
    last = [clock_seq[0]]

    def clock(h, which):
        assert h == "gpu0" and which == 1
        try:
            last[0] = next(it)
        except StopIteration:
            pass
        return last[0]
    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetMaxClockInfo = lambda h, which: 1965
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reason_bits
    return nv


def test_clock_sampler_reports_median_and_reasons(monkeypatch):
    nv = _fake_nvml([1965, 1950, 1965, 1900, 1965], 0x4)
    c = bench.Clocks(device=None)

    def handle(self):
        self.nv = nv
        return "gpu0"
    monkeypatch.setattr(bench.Clocks, "_handle", handle)
    c.start()
    time.sleep(0.1)
    r = c.stop()
    assert r["sm_max_mhz"] == 1965 and r["samples"] >= 3
    assert r["sm_mhz"] in (1950, 1965)
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_sampler_reports_why_it_is_unavailable(monkeypatch):
    def handle(self):
        raise RuntimeError("no NVML here")
    monkeypatch.setattr(bench.Clocks, "_handle", handle)
    c = bench.Clocks(device=None)
    c.start()
    r = c.stop()
    assert "unavailable" in r and "no NVML" in r["unavailable"]


def test_ncu_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    """A captured DRAM-traffic figure is reported only while the kernel's source file still
    hashes to the value recorded with it."""
    import hashlib
    fake = tmp_path / "block_diffusion_lm_masked_b200" / "csrc"
    fake.mkdir(parents=True)
    (fake / "k_x.cu").write_text("// a kernel\n")
    digest = hashlib.sha256((fake / "k_x.cu").read_bytes()).hexdigest()[:16]
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {("w", "kern"): ("k_x.cu", digest, 123.0e6)})
    assert bench._ncu_traffic("w", "kern") == pytest.approx(123.0e6)
    assert bench._ncu_traffic("w", "other") is None                    # no capture for it
    assert bench._ncu_traffic("v", "kern") is None
    with open(fake / "k_x.cu", "a") as f:
        f.write("\n// changed\n")
    assert bench._ncu_traffic("w", "kern") is None                     # the kernel changed since


def test_recorded_traffic_names_existing_sources():
    for (workload, kernel), (src, digest, nbytes) in bench.NCU_TRAFFIC.items():
        assert os.path.exists(os.path.join(ROOT, "block_diffusion_lm_masked_b200", "csrc", src)), src
        assert len(digest) == 16 and nbytes > 0


def test_peaks_fall_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    hbm, tf, tfs, src = bench._peaks()
    assert src == "fallback" and hbm == 6650.0 and tf == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6554.6, "bf16_tflops": 1591.5}')
    hbm, tf, tfs, src = bench._peaks()
    assert src == "measured" and hbm == 6554.6 and tf == tfs == 1591.5


def test_job_value_counts_every_rank_over_the_slowest():
    assert bench.job_value(1, 256, 1000, 347.6) == pytest.approx(256 * 1000 / 0.3476)
    assert bench.job_value(8, 256, 1000, 400.0) == pytest.approx(8 * 256 * 1000 / 0.4)


def test_attention_kind_follows_the_switch(monkeypatch):
    monkeypatch.delenv("DG_ATTN_PAIR", raising=False)
    assert bench._attention_kind().startswith("one head")
    monkeypatch.setenv("DG_ATTN_PAIR", "1")
    assert bench._attention_kind().startswith("head pairs")
    monkeypatch.setenv("DG_ATTN_PAIR", "0")
    assert bench._attention_kind().startswith("one head")


class _FakeSampler:
    """Stands in for bench.Clocks: each region's record comes from a script."""
    script = []

    def __init__(self, dev):
        self.dev = dev

    def start(self):
        pass

    def stop(self):
        reasons = _FakeSampler.script.pop(0)
        return {"sm_mhz": 1900.0, "sm_max_mhz": 1965, "reasons": reasons, "samples": 10}


@pytest.fixture
def one_rank(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    return bench.Ranks("gloo", device="cpu")


def _count_runs():
    runs = []

    def run():
        runs.append(len(runs))
        return ("result", len(runs))
    return runs, run


@pytest.mark.parametrize("reasons", [[], ["sw_power_cap"]])
def test_clean_or_power_capped_region_is_kept(one_rank, reasons):
    r = one_rank
    _FakeSampler.script = [list(reasons)]
    runs, run = _count_runs()
    out, clocks = bench.clocked(r, "cpu", run, sampler=_FakeSampler)
    assert runs == [0] and out == ("result", 1)
    assert clocks["reasons"] == reasons and "remeasured_after" not in clocks


@pytest.mark.parametrize("bad", ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"])
def test_slowed_region_is_timed_once_more(one_rank, bad):
    r = one_rank
    _FakeSampler.script = [["sw_power_cap", bad], ["sw_power_cap"]]
    runs, run = _count_runs()
    out, clocks = bench.clocked(r, "cpu", run, sampler=_FakeSampler)
    assert runs == [0, 1] and out == ("result", 2)      # the second region's result and clocks
    assert clocks["reasons"] == ["sw_power_cap"] and clocks["remeasured_after"] == [bad]
    assert _FakeSampler.script == []


def test_second_slowed_region_is_reported_not_retried(one_rank):
    r = one_rank
    _FakeSampler.script = [["hw_slowdown"], ["hw_slowdown"]]
    runs, run = _count_runs()
    _, clocks = bench.clocked(r, "cpu", run, sampler=_FakeSampler)
    assert runs == [0, 1] and clocks["reasons"] == ["hw_slowdown"]   # once more, not again
