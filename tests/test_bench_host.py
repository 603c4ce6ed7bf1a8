"""Host-side pieces of bench.py that need no GPU: the DRAM-traffic figures are
taken from profiles/traffic.json only while the kernel's sources are the ones
the counters were captured on, and only for the workload they describe."""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_digests_match_the_current_sources():
    t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for kernel, e in t["kernels"].items():
        assert bench._source_digest(e["sources"]) == e["sha256"], (
            f"{kernel}: its sources changed since the counters were captured; capture again")
        assert bench._traffic_from_profiles(kernel, t["workload"]) == e["bytes_per_launch"]


def test_traffic_is_withheld_for_another_workload_or_unknown_kernel():
    t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for some in t["kernels"]:
        assert bench._traffic_from_profiles(some, "another_workload") is None
    assert bench._traffic_from_profiles("no_such_kernel", t["workload"]) is None


def test_source_digest_depends_on_names_and_bytes():
    a = bench._source_digest(["sm100.cuh", "conv.cuh"])
    assert a != bench._source_digest(["conv.cuh", "sm100.cuh"])
    assert a == bench._source_digest(["sm100.cuh", "conv.cuh"])
