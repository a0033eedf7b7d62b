"""Host logic of bench.py that needs no GPU: the roofline denominators read from
the generated peaks file (each missing or malformed entry falls back to
the earlier measurement), and the argument checks of the timing contract."""
import json

import pytest

import bench


@pytest.fixture()
def peaks_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path / "MEASURED_PEAKS.json"


def test_peaks_absent_fall_back(peaks_file):
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks == bench.FALLBACK_PEAKS


def test_peaks_measured(peaks_file):
    peaks_file.write_text(json.dumps({"hbm_gbs": 6547, "bf16_tflops": 1630,
                                      "bf16_tflops_sustained": 1383.8, "clocks": {"sm": 1965}}))
    peaks, kind = bench.load_peaks()
    assert kind == "measured"
    assert peaks == {"hbm_gbs": 6547.0, "bf16_tflops": 1630.0, "bf16_tflops_sustained": 1383.8}


@pytest.mark.parametrize("content,kind", [
    ('{"hbm_gbs": 6547}', "partly measured"),
    ('{"hbm_gbs": "6547", "bf16_tflops": -1, "bf16_tflops_sustained": true}', "fallback"),
    ("not json", "fallback"),
    ("[1, 2]", "fallback"),
])
def test_peaks_malformed_entries_fall_back(peaks_file, content, kind):
    peaks_file.write_text(content)
    peaks, got = bench.load_peaks()
    assert got == kind
    for key, v in peaks.items():
        assert isinstance(v, float) and v > 0, key


def test_timing_contract_arguments():
    assert bench.parse([]).warmup >= 3
    with pytest.raises(SystemExit):
        bench.parse(["--warmup", "2"])


def test_clock_reasons_from_nvml_bits():
    assert bench.ClockSampler.reasons_of(0) == []
    assert bench.ClockSampler.reasons_of(0x4) == ["sw_power_cap"]
    assert bench.ClockSampler.reasons_of(0x4 | 0x8 | 0x20 | 0x40 | 0x80) == [
        "sw_power_cap", "hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown",
        "hw_power_brake_slowdown"]
    assert bench.ClockSampler.reasons_of(0x1 | 0x2) == []   # idle, application clocks


def test_clock_sampler_without_a_gpu_reports_no_clock():
    c = bench.ClockSampler(0)
    c.start()
    out = c.stop()
    assert out["sm_mhz"] is None or out["sm_mhz"] > 0
    assert "reasons" in out
