"""Host-side pieces of bench.py, on CPU: the clock summary keeps only the
samples of the timed region and reports every throttle reason it saw; the
in-process NVML sampler (driven here by a fake NVML module, read-only
queries) feeds the same summary and falls back when NVML fails; the
DRAM traffic figure is taken from the committed profile only while the
profiled source is unchanged; the reported config names the workload."""
import hashlib
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mla_latent_kv_33_b200 import synth  # noqa: E402


def _line(sm, smax=1965, reasons=("Not Active",) * 4):
    return f"0, {sm}, {smax}, 700.00, 0x0, " + ", ".join(reasons) + "\n"


def test_clock_summary_keeps_the_timed_window():
    c = bench.ClockSampler("0")
    c.samples = [(0.0, _line(1200)), (1.0, _line(1965)), (1.1, _line(1950)), (1.2, _line(1965)), (3.0, _line(900))]
    c.mark(0.95, 1.25)
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["samples"] == 3 and s["reasons"] == []


def test_clock_summary_reports_throttle_reasons():
    c = bench.ClockSampler("0")
    c.samples = [(1.0, _line(1400, reasons=("Not Active", "Not Active", "Not Active", "Active"))),
                 (1.1, _line(1300, reasons=("Active", "Not Active", "Not Active", "Not Active")))]
    c.mark(0.9, 1.2)
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_summary_short_region_takes_the_nearest_sample():
    c = bench.ClockSampler("0")
    c.samples = [(0.0, _line(1000)), (1.0, _line(1800)), (2.0, _line(1100))]
    c.mark(1.001, 1.002)  # shorter than the sampling period
    s = c.summary()
    assert s["samples"] == 1 and s["sm_mhz"] == 1800.0


def test_clock_summary_without_samples():
    c = bench.ClockSampler("0")
    c.samples = [(1.0, "garbage\n")]
    assert c.summary() is None


def test_decode_traffic_follows_the_profiled_source(tmp_path, monkeypatch):
    got = bench.decode_traffic("v2_b64_paged")
    doc = open(os.path.join(ROOT, "profiles", "k_decode_v2_b64_paged.md")).read()
    src = open(os.path.join(ROOT, "mla_latent_kv_33_b200", "csrc", "decode_tc.cuh"), "rb").read()
    fields = dict(l.split(": ", 1) for l in doc.splitlines() if ": " in l and l.split(": ", 1)[0] in
                  ("traffic_bytes_per_launch", "decode_source_sha256_16"))
    if fields["decode_source_sha256_16"].strip() == hashlib.sha256(src).hexdigest()[:16]:
        assert got == int(fields["traffic_bytes_per_launch"])
    else:
        assert got is None
    assert bench.decode_traffic("no_such_workload") is None


def test_config_names_the_workload():
    w = synth.shrink(synth.WORKLOADS["v2_b64_paged"], B=3, L_lo=5, L_hi=130, d=64, d_cq=32)
    x = synth.generate(w)
    cfg = bench.config_of(w, 1, x)
    assert cfg["workload"] == "v2_b64_paged" and cfg["batch"] == 3 and cfg["paged"] is True
    assert cfg["seq_len_min"] == int(np.min(x.seq_lens)) and cfg["parallelism"] == "replicas1"
    assert "model" not in cfg


def test_percentiles_of_step_durations():
    ms = [0.1 * k for k in range(1, 101)]  # 0.1 .. 10 ms
    p10, p50, p90 = bench.percentiles_us(ms)
    assert abs(p10 - 1090.0) < 1e-6 and abs(p50 - 5050.0) < 1e-6 and abs(p90 - 9010.0) < 1e-6


class _FakeNVML:
    """The few read-only NVML entry points the sampler calls, with made-up
    reason bits; counts init/shutdown so that the test sees them paired."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 1 << 0
    nvmlClocksEventReasonHwThermalSlowdown = 1 << 1
    nvmlClocksEventReasonSwThermalSlowdown = 1 << 2
    nvmlClocksEventReasonSwPowerCap = 1 << 3

    def __init__(self, fail_queries=False):
        self.fail_queries = fail_queries
        self.inits = self.shutdowns = self.queries = 0
        self.handle_of = None

    def nvmlInit(self):
        self.inits += 1

    def nvmlShutdown(self):
        self.shutdowns += 1

    def nvmlDeviceGetHandleByUUID(self, uuid):
        self.handle_of = uuid
        return "h"

    def nvmlDeviceGetHandleByIndex(self, i):
        self.handle_of = i
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        assert h == "h" and kind == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        if self.fail_queries:
            raise RuntimeError("not supported")
        self.queries += 1
        return 1965 if self.queries % 2 else 1950

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.nvmlClocksEventReasonSwPowerCap

    def nvmlDeviceGetPowerUsage(self, h):
        return 700000  # milliwatts


def test_nvml_sampler_fills_the_timed_window():
    fake = _FakeNVML()
    with bench.ClockSampler("GPU-0000", nvml=fake) as c:
        a = time.perf_counter()
        time.sleep(0.04)
        c.mark(a, time.perf_counter())
    assert fake.handle_of == "GPU-0000" and fake.inits == 1 and fake.shutdowns == 1
    s = c.summary()
    assert s["samples"] >= 5 and s["sm_max_mhz"] == 1965.0
    assert 1950.0 <= s["sm_mhz"] <= 1965.0 and s["reasons"] == ["sw_power_cap"]


def test_nvml_sampler_falls_back_when_queries_fail():
    fake = _FakeNVML(fail_queries=True)
    with bench.ClockSampler("3", nvml=fake) as c:
        assert c.poller is None  # handed over to the nvidia-smi path
    assert fake.handle_of == 3 and fake.inits == 1 and fake.shutdowns == 1


def test_profile_summaries_leave_clocks_alone_and_parse():
    """Every ncu command a summary records runs with --clock-control none, and
    each decode summary carries the two fields the bench reads."""
    pdir = os.path.join(ROOT, "profiles")
    for name in sorted(os.listdir(pdir)):
        text = open(os.path.join(pdir, name)).read()
        # an ncu command may continue over backslash-ended lines
        cmds = text.replace("\\\n", " ").splitlines()
        for c in cmds:
            if c.lstrip().startswith("ncu "):
                assert "--clock-control none" in c, (name, c)
        if name.startswith("k_decode_"):
            fields = dict(l.split(": ", 1) for l in text.splitlines()
                          if l.startswith(("traffic_bytes_per_launch:", "decode_source_sha256_16:")))
            assert int(fields["traffic_bytes_per_launch"]) > 0 and len(fields["decode_source_sha256_16"].strip()) == 16
