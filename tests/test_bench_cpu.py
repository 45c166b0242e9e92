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
    got = bench.ncu_traffic(I.WAN_FFN.name, "qgemm_kernel")
    if d["source_hash"] == bench.kernel_source_hash():
        assert got == d["workloads"][I.WAN_FFN.name]["qgemm_kernel"]["dram_bytes_per_launch_full"]
    else:  # the kernels changed since the counters were taken: no stale number
        assert got is None
    assert bench.ncu_traffic("no such workload", "qgemm_kernel") is None
