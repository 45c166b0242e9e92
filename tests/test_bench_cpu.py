"""Host logic of bench.py that needs no GPU: workload selection and the
committed ncu traffic lookup."""

import json
import os

import pytest

import bench
from bit_quantized_linear_hadamard_b200 import inputs as I


def test_workload_names():
    assert bench.workload_config(I, None) is I.WAN_FFN
    assert bench.workload_config(I, "w4a4") is I.WAN_FFN
    assert bench.workload_config(I, "w8a8") is I.WAN_FFN_W8
    assert bench.workload_config(I, "w4a8").act_bits == 8
    assert bench.workload_config(I, "w4a6").act_bits == 6
    assert bench.workload_config(I, I.WAN_FFN_W4A6.name) is I.WAN_FFN_W4A6
    with pytest.raises(SystemExit):
        bench.workload_config(I, "w2a2")


def test_traffic_lookup_follows_the_kernel_sources():
    path = os.path.join(bench.PROFILES, "ncu_traffic.json")
    with open(path) as f:
        d = json.load(f)
    for kernel in ("qgemm_kernel", "rotate_quant_kernel"):
        got = bench.ncu_traffic(I.WAN_FFN.name, kernel)
        if d["source_hashes"][kernel] == bench.kernel_source_hash(kernel):
            assert got == d["workloads"][I.WAN_FFN.name][kernel]["dram_bytes_per_launch_full"]
        else:  # the kernel changed since its counters were taken: no stale number
            assert got is None
    assert bench.ncu_traffic("no such workload", "qgemm_kernel") is None
    assert bench.ncu_traffic(I.WAN_FFN.name, "no such kernel") is None


def test_traffic_of_one_kernel_survives_a_change_to_the_other(monkeypatch):
    path = os.path.join(bench.PROFILES, "ncu_traffic.json")
    with open(path) as f:
        d = json.load(f)
    rec = dict(d["source_hashes"])
    monkeypatch.setattr(bench, "kernel_source_hash",
                        lambda kernel=None: "changed" if kernel == "qgemm_kernel" else rec[kernel])
    assert bench.ncu_traffic(I.WAN_FFN.name, "qgemm_kernel") is None
    assert bench.ncu_traffic(I.WAN_FFN.name, "rotate_quant_kernel") == \
        d["workloads"][I.WAN_FFN.name]["rotate_quant_kernel"]["dram_bytes_per_launch_full"]


def test_clock_sampler_reports_the_timed_region_from_nvml(monkeypatch):
    """The clock record comes from NVML reads taken between the marks around
    the timed region: samples before and after it (idle clocks, another
    reason) are not reported; reason bits map to their names."""
    import sys
    import time
    import types

    import bench

    state = {"clock": 900, "reasons": 0x1}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0, nvmlInit=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda u: "h", nvmlDeviceGetHandleByIndex=lambda i: "h",
        nvmlDeviceGetClockInfo=lambda h, c: state["clock"],
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: state["reasons"],
        nvmlDeviceGetPowerUsage=lambda h: 700000)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.03)
    state.update(clock=1965, reasons=0x4)
    s.mark_start()
    time.sleep(0.05)
    s.mark_end()
    time.sleep(0.01)
    state.update(clock=600, reasons=0x8 | 0x40)
    time.sleep(0.02)
    r = s.stop()
    assert r["source"].startswith("nvml") and "timed region" in r["source"]
    assert r["sm_mhz"] == 1965 and r["sm_max_mhz"] == 1965 and r["power_w_max"] == 700.0
    assert r["reasons"] == ["sw_power_cap"] and r["samples"] >= 5
