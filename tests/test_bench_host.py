"""Host logic of bench.py, checked without a GPU: the clock record (NVML
samples taken during the timed loop, nvidia-smi samples beside them, the
clock-event reason bits), and the traffic figures read from profiles/ only for
the source they were captured on."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _FakeSmi(out):
    """A ClockSampler whose nvidia-smi run printed `out`."""
    smi = bench.ClockSampler.__new__(bench.ClockSampler)
    smi.proc, smi.out = object(), out
    return smi


def _fast(samples, max_mhz=1965, err=None):
    f = bench.NvmlSampler.__new__(bench.NvmlSampler)
    f.samples, f.max_mhz, f.err = samples, max_mhz, err
    return f


SMI_ROWS = ("0, 1965, 1965, 900.1, 100, 0x0, Not Active, Not Active, Not Active, Not Active\n"
            "0, 1800, 1965, 1000.0, 100, 0x4, Not Active, Not Active, Not Active, Active\n"
            "0, 345, 1965, 120.0, 0, 0x0, Not Active, Not Active, Not Active, Not Active\n")


def test_nvml_samples_give_the_record():
    # 0x4 sw_power_cap, 0x8 hw_slowdown, 0x20 sw_thermal, 0x40 hw_thermal
    f = _fast([(1965, 0x0), (1950, 0x4), (1900, 0x4 | 0x40), (1965, 0x0)])
    r = bench.clock_record(f, _FakeSmi(SMI_ROWS))
    assert r["sm_mhz"] == 1957.5 and r["sm_min_mhz"] == 1900 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert r["samples"] == 4 and r["source"].startswith("nvml")
    # nvidia-smi's own summary rides along: only samples under load count.
    smi = r["nvidia_smi"]
    assert smi["samples"] == 3 and smi["samples_under_load"] == 2
    assert smi["sm_mhz"] == 1882.5 and smi["reasons"] == ["sw_power_cap"]


def test_without_nvml_samples_nvidia_smi_is_the_record():
    r = bench.clock_record(_fast([], err="nvml unavailable: NVMLError"), _FakeSmi(SMI_ROWS))
    assert r["source"].startswith("nvidia-smi") and r["nvml"] == "nvml unavailable: NVMLError"
    assert r["sm_mhz"] == 1882.5 and r["reasons"] == ["sw_power_cap"]


def test_no_sampler_at_all():
    smi = bench.ClockSampler.__new__(bench.ClockSampler)
    smi.proc = None
    r = bench.clock_record(_fast([]), smi)
    assert r["sm_mhz"] is None and r["reasons"] == ["nvidia-smi unavailable"]


def test_nvml_sampler_without_a_device_records_why():
    # No GPU in this container: the sampler says so and takes no samples.
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    f = bench.NvmlSampler(torch.device("cuda", 0))
    f.start()
    f.stop()
    assert f.summary() is None and f.err and f.err.startswith("nvml unavailable")


def test_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    sha = bench.source_sha("fwd_tc.cu", "fwd_moments.cu", "polar_common.cuh", "tc_common.cuh",
                           "bwd_coef.cuh")
    assert len(sha) == 16
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(
        '{"prefill": {"source_sha": "%s", "dram_bytes_per_launch": 123}}' % sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("prefill", sha) == 123
    assert bench.profiled_traffic("prefill", "0" * 16) is None  # the kernel changed since
    assert bench.profiled_traffic("decode", sha) is None          # never captured
