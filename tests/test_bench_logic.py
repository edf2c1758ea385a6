"""Host logic of bench.py (no GPU): workload selection, the launch count it
claims per step, the roofline it reports against, and the recorded ncu
traffic lookup."""
import json
import os

import pytest

import bench
from nvfp4_expert_layer_b200 import workloads as W


class _Args:
    def __init__(self, workload):
        self.workload = workload


def test_workload_names():
    assert bench.workload_names(_Args("all")) == bench.ALL
    assert bench.workload_names(_Args("decode1")) == ("decode1",)
    assert bench.workload_names(_Args("decode64,verify")) == ("decode64", "verify")


@pytest.mark.parametrize("name,thr,expected", [
    # small batches: the router kernel (top-k and permutation in its last block),
    # the 1..8-row light kernel, the combine
    ("decode1", 9, 3), ("tiny", 9, 3),
    # 33..2048 pairs, T <= 256: router, top-k, 3 permutation kernels; the dense
    # class (quantiser, gather, 2 GEMMs); only the 1..8-row light kernel can
    # have jobs at thr = 9; the combine
    ("decode64", 9, 11), ("verify", 9, 11),
    # every expert light: the 9..16- and 17..32-row kernels too
    ("decode64", 128, 9),
    # T = thr: the dense-class kernels launch (and find no expert with 128 rows)
    # besides the three light kernels
    ("verify", 128, 13),
    # T > 256: weight split, tensor-core router, x staging, top-k, 3 permutation kernels
    ("prefill", 9, 13),
])
def test_launches_per_step(name, thr, expected):
    assert bench.launches_per_step(W.CONFIGS[name], thr) == expected


def test_roofline_choice():
    # prefill: ~512 rows per expert, above the ridge point; decode: a few rows
    assert bench.tensor_bound(W.CONFIGS["prefill"], 256)
    assert not bench.tensor_bound(W.CONFIGS["decode64"], 53)
    assert not bench.tensor_bound(W.CONFIGS["verify"], 224)
    assert not bench.tensor_bound(W.CONFIGS["decode1"], 8)


def test_recorded_traffic_lookup():
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(path) as fh:
        rec = json.load(fh)
    for key, ent in rec.items():
        kernel, workload = key.split("@")
        got = bench.recorded_traffic(kernel, workload)
        # valid only while the kernel's sources match the digest taken with the counters
        if ent["source_digest"] == bench.source_digest(kernel):
            assert got == ent["dram_bytes_per_launch"]
        else:
            assert got is None
    assert bench.recorded_traffic("expert_kernel", "no-such-workload") is None
