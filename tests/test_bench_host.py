"""Host-side logic of bench.py on the CPU: the clock sampler (against a fake
NVML), the reasons it decodes, and how it finds the timed GPU in NVML."""
import sys
import time
import types

import pytest
import torch

import bench


def _fake_nvml(calls, reasons_bits=0x4 | 0x20, mhz=1500):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlInit = lambda: None

    def by_uuid(u):
        calls.append(("uuid", u))
        return "handle"

    def by_index(i):
        calls.append(("index", i))
        return "handle"

    m.nvmlDeviceGetHandleByUUID = by_uuid
    m.nvmlDeviceGetHandleByIndex = by_index
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    m.nvmlDeviceGetClockInfo = lambda h, c: mhz
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons_bits
    return m


def _sample(seconds=0.04):
    with bench.ClockSampler(0) as c:
        time.sleep(seconds)
    return c.summary()


def test_sampler_finds_the_gpu_by_uuid_and_decodes_reasons(monkeypatch):
    calls = []
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(calls))
    props = types.SimpleNamespace(uuid="58a9c8b1-6ad7-1234-5678-9abcdef01234")
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: props)
    s = _sample()
    assert calls[0] == ("uuid", "GPU-58a9c8b1-6ad7-1234-5678-9abcdef01234")
    assert s["nvml_device_by"] == "uuid"
    assert s["sm_mhz"] == 1500 and s["sm_max_mhz"] == 1965 and s["samples"] >= 2
    assert s["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]


def test_sampler_falls_back_to_the_index(monkeypatch):
    calls = []
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(calls, reasons_bits=0))

    def no_props(i):
        raise RuntimeError("no CUDA device")

    monkeypatch.setattr(torch.cuda, "get_device_properties", no_props)
    s = _sample()
    assert calls[0] == ("index", 0)
    assert s["nvml_device_by"] == "index" and s["reasons"] == []


def test_sampler_without_nvml_reports_why(monkeypatch):
    m = types.ModuleType("pynvml")

    def fail():
        raise OSError("NVML library not found")

    m.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", m)
    s = _sample(0.0)
    assert s["sm_mhz"] is None
    assert "nvml unavailable" in s["reasons"][0]


@pytest.mark.parametrize("world,flops,ms,expect", [(1, 2e12, 1.0, 2000.0), (4, 1e12, 2.0, 2000.0)])
def test_job_throughput_counts_all_ranks_over_the_slowest(world, flops, ms, expect):
    assert bench.job_tflops(world, flops, ms) == pytest.approx(expect)


def test_recorded_traffic_only_for_the_captured_kernel(monkeypatch):
    """The GEMM's recorded DRAM traffic is reported only for the full-size
    prefill workload and only while the kernel sources hash to the value
    recorded with the capture."""
    args = types.SimpleNamespace(workload="prefill", x_rows=0)
    monkeypatch.setitem(bench.GEMM_PREFILL_TRAFFIC, "kernel_sources_sha1", bench.gemm_sources_sha1())
    assert bench.recorded_traffic(args)["bytes"] == bench.GEMM_PREFILL_TRAFFIC["bytes"]
    assert bench.recorded_traffic(types.SimpleNamespace(workload="prefill", x_rows=8192)) is None
    assert bench.recorded_traffic(types.SimpleNamespace(workload="mlp8b", x_rows=0)) is None
    monkeypatch.setitem(bench.GEMM_PREFILL_TRAFFIC, "kernel_sources_sha1", "0" * 40)
    assert bench.recorded_traffic(args) is None


def test_x_rows_replaces_only_the_activation_rows():
    wl = bench.workload_of(types.SimpleNamespace(workload="prefill", x_rows=8192))
    ref = bench.workloads.WORKLOADS["prefill"]
    assert (wl.M, wl.N, wl.K) == (8192, ref.N, ref.K)
    assert wl.x.seed == ref.x.seed and wl.w == ref.w
