"""Host-side accounting of the benchmark, checked without a GPU: the
algorithmic bytes per kernel against the per-workload figures the design
states (read each input once, write each output once, indices included), the
peak fallback, the profiled-traffic guard and the config keys of the JSON
line."""
import argparse
import json
import os

import pytest

import bench
from dispatch_moonep_plan_b200 import workloads as wl


@pytest.mark.parametrize("name,dispatch_mb,combine_mb", [
    # T*H*2 + P*row + 4P  and  P*H*2 + T*H*2 + 8P, in units of 10^6 bytes
    ("uniform", 32768 * 2048 * 2 + 196608 * 4096 + 4 * 196608,
     196608 * 4096 + 32768 * 4096 + 8 * 196608),
    ("zipf", 32768 * 7168 * 2 + 262144 * 14336 + 4 * 262144,
     262144 * 14336 + 32768 * 14336 + 8 * 262144),
    ("hot", 262144 * 7168 * 2 + 2097152 * 14336 + 4 * 2097152,
     2097152 * 14336 + 262144 * 14336 + 8 * 2097152),
    # fp8 rows: 4096 code bytes + 32 fp32 scales
    ("fp8", 262144 * 4096 * 2 + 2097152 * (4096 + 128) + 4 * 2097152,
     2097152 * 8192 + 262144 * 8192 + 8 * 2097152),
])
def test_algorithmic_bytes(name, dispatch_mb, combine_mb):
    b = bench.algorithmic_bytes(wl.WORKLOADS[name])
    assert b["dispatch"] == dispatch_mb
    assert b["combine"] == combine_mb
    P = wl.WORKLOADS[name]["R"] * wl.WORKLOADS[name]["S"] * wl.WORKLOADS[name]["K"]
    assert b["plan"] == 12 * P


def test_peaks_measured_or_fallback():
    peak, kind = bench.peaks()
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        assert kind == "measured" and peak == float(json.load(open(path))["hbm_gbs"])
    else:
        assert kind == "fallback" and peak == 6650.0
    burst, sustained, kind2 = bench.tensor_peaks()
    assert burst >= sustained > 0 and kind2 == kind


def test_profiled_traffic_only_for_the_current_source():
    d = json.load(open(bench.PROFILE_TRAFFIC))
    for key, v in d.items():
        kernel, workload = key.split("/", 1)
        got = bench.profiled_traffic(kernel, workload)
        if v["source_sha"] == bench.kernel_source_hash(v["source"]):
            assert got == v["dram_bytes_per_launch"] == v["read"] + v["write"]
        else:
            assert got is None
    assert bench.profiled_traffic("combine", "no-such-workload") is None


def test_workload_config_keys():
    args = argparse.Namespace(rule=1, alpha=None)
    c = bench.workload_config(wl.WORKLOADS["zipf"], args)
    assert c["workload"] == wl.WORKLOADS["zipf"]["name"] and c["rule"] == 1
    assert c["alpha"] == wl.WORKLOADS["zipf"]["alpha"]
    assert "flushed" in c["l2"]
    assert "model" not in c  # the config names a workload, not a model
    c = bench.workload_config(wl.WORKLOADS["uniform"], argparse.Namespace(rule=0, alpha=None))
    assert c["sigma"] == wl.WORKLOADS["uniform"]["sigma"]


def test_cli_rejects_short_warmup(capsys):
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
