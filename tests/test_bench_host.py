"""Host-side pieces of bench.py that need no GPU: the clock sampler (against
a fake NVML), and the lookup of a committed per-launch DRAM traffic record."""
import json

import bench


class _FakeNVML:
    NVML_CLOCK_SM = 1

    def __init__(self, mhz=1900, mask=0x4, fail=False):
        self.mhz, self.mask, self.fail = mhz, mask, fail

    def nvmlDeviceGetMaxClockInfo(self, h, clock):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, clock):
        if self.fail:
            raise RuntimeError("NVML gone")
        return self.mhz

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.mask


def _counting(n):
    state = {"k": 0}

    def busy():
        state["k"] += 1
        return state["k"] <= n
    return busy


def test_clock_sampler_samples_while_the_region_drains(monkeypatch):
    nv = _FakeNVML(mhz=1900, mask=0x4 | 0x8)  # sw_power_cap + hw_slowdown
    monkeypatch.setattr(bench.ClockSampler, "_nvml_handle", lambda self: (nv, object()))
    with bench.ClockSampler(0) as c:
        c.sample_while(_counting(5))
    s = c.summary()
    assert s["samples"] >= 5
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_sampler_survives_a_failing_nvml(monkeypatch):
    nv = _FakeNVML(fail=True)
    monkeypatch.setattr(bench.ClockSampler, "_nvml_handle", lambda self: (nv, object()))
    with bench.ClockSampler(0) as c:
        c.sample_while(_counting(3))  # must not raise
    assert c.summary()["samples"] == 0


def test_clock_sampler_without_nvml_reports_no_samples(monkeypatch):
    def no_nvml(self):
        raise ImportError("no NVML here")
    monkeypatch.setattr(bench.ClockSampler, "_nvml_handle", no_nvml)
    monkeypatch.setattr(bench.ClockSampler, "_start_smi", lambda self: None)
    with bench.ClockSampler(0) as c:
        c.sample_while(_counting(3))  # no-op without NVML
    s = c.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None


def test_traffic_record_is_used_only_for_the_current_kernel_source(tmp_path, monkeypatch):
    digest = "d1"
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"kernel": "lora_gemm_fwd", "workload": "w", "dram_bytes_per_launch": 123}
    (prof / "k.md").write_text(
        "summary text\n"
        "traffic_record: " + json.dumps(dict(rec, source_digest=digest)) + "\n"
        "traffic_record: " + json.dumps(dict(rec, workload="other", source_digest="old")) + "\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "gemm_source_digest", lambda: digest)
    assert bench.recorded_traffic("lora_gemm_fwd", "w") == 123
    assert bench.recorded_traffic("lora_gemm_fwd", "other") is None  # taken on older source
    assert bench.recorded_traffic("lora_gemm_dx", "w") is None
    monkeypatch.setattr(bench, "gemm_source_digest", lambda: "d2")
    assert bench.recorded_traffic("lora_gemm_fwd", "w") is None  # kernel changed since
