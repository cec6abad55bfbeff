"""Host-side helpers of bench.py: the shared config object (identical in both
arms), the byte accounting, the profiled-traffic lookup (only for the captured
workload and the captured kernel source)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_kv_cache_15_b200 import workloads as W  # noqa: E402


def test_both_arms_describe_the_workload_alike():
    w = W.make_workload(5, "full")
    c = bench.workload_config(w, w.n_layers, 1)
    assert c == bench.workload_config(W.make_workload(5, "full"), w.n_layers, 1)
    assert c["workload"] == w.name and c["batch"] == w.batch and c["layers"] == w.n_layers
    assert c["tail"] == w.tail and c["rotation"] == "varnorm+hadamard-128"
    assert c["step"].startswith("per layer: append 2048 token(s) x 8 seq(s)")
    assert c["l2"].startswith("no flush")


def test_tiny_workload_is_timed_with_l2_flushes():
    assert "flushed" in bench.l2_note(W.make_workload(1, "full"))
    for cfg in (2, 3, 4, 5):
        assert bench.l2_note(W.make_workload(cfg, "full")).startswith("no flush")


def test_byte_accounting_matches_the_documented_row_sizes():
    w = W.make_workload(2, "full")
    assert bench.token_head_bytes(w, 0) == 8 * (136 + 72)
    # one decode launch of the Llama-shaped layer: 32768 tokens x 8 heads x 208 B + q + out
    assert bench.decode_bytes(w, 0, [32768]) == 32768 * 8 * 208 + 32 * 128 * 6
    w5 = W.make_workload(5, "full")
    raw = 8 * 2 * 256
    # a 2048-token chunk into a sequence longer than its 256-token tail: 2048 input rows
    # read, 256 ring rows read and requantized, 1792 pass straight through, 256 enter the ring
    assert bench.append_bytes(w5, 0, 5000, 2048) == 2048 * raw + 256 * raw + 2048 * 8 * 144 + 256 * raw
    w4 = W.make_workload(4, "full")
    r, b = w4.rank[0][0], w4.k_bits[0][0]
    assert bench.row_bytes(W.RANK, r, b) == r * b // 8 + 2 * ((r + 31) // 32)


def test_profiled_traffic_is_reported_only_for_its_workload():
    # only a capture of the workload, with the current decode source, is used
    for cfg in (1, 2, 3, 4, 5):
        t = bench.traffic_from_profile(W.make_workload(cfg, "full").name)
        assert t is None or t > 0


def test_kernel_source_hash_covers_the_decode_sources():
    h = bench.kernel_source_sha256()
    assert len(h) == 64
    for name in bench.DECODE_SOURCES:
        assert os.path.exists(os.path.join(ROOT, "quantized_kv_cache_15_b200", "csrc", name))


def test_decode_multiply_adds():
    """A decode launch's multiply-adds: per visible (token, kv head), G query heads x
    (score + value) x the head's stored width (128, or the rank of a projected head)."""
    import bench
    from quantized_kv_cache_15_b200 import workloads as W
    w = W.make_workload(1, "full")                                   # 1024 tokens, 2 kv heads, G = 4
    assert bench.decode_macs(w, 0, w.ctx) == 1024 * 4 * 2 * (2 * 128)
    w4 = W.make_workload(4, "full")
    assert bench.decode_macs(w4, 3, [100]) == 100 * w4.G * 2 * sum(w4.rank[3])
    assert 36.0 < bench.DP2A_PEAK_TMACS < 38.0
