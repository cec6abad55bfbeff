"""Host-side helpers of bench.py: the shared config object, the profiled-traffic
lookup (only for the captured workload and the captured kernel source) and the
oracle baseline's scaling to the step."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_kv_cache_15_b200 import workloads as W  # noqa: E402


def test_both_arms_describe_the_workload_alike():
    w = W.make_workload(5, "full")
    c = bench.workload_config(w, w.n_layers, 1, "x")
    assert c["workload"] == w.name and c["batch"] == w.batch and c["layers"] == w.n_layers
    assert c["tail"] == w.tail and c["rotation"] == "varnorm+hadamard-128"
    assert c["step"].startswith("per layer: append 2048 token(s) x 8 seq(s)")


def test_profiled_traffic_is_reported_only_for_its_workload():
    w2 = W.make_workload(2, "full").name
    t = bench.traffic_from_profile(w2)
    # the committed capture covers the llama8b workload; a stale kernel hash gives None
    assert t is None or t > 54_000_000
    for cfg in (1, 3, 4, 5):
        assert bench.traffic_from_profile(W.make_workload(cfg, "full").name) is None


def test_kernel_source_hash_covers_the_decode_sources():
    h = bench.kernel_source_sha256()
    assert len(h) == 64
    for name in bench.DECODE_SOURCES:
        assert os.path.exists(os.path.join(ROOT, "quantized_kv_cache_15_b200", "csrc", name))
