"""Host-side pieces of bench.py that need no GPU: the oracle timings of the
cpu_baseline object and the DRAM-traffic lookup."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402


def test_oracle_extras_tiny_workload():
    oracle.build()
    w = synth.WORKLOADS["tiny"]
    x, s = synth.gen_layer_inputs(w, 0)
    r = bench.oracle_extras(w, x, s, w.seed(0))
    assert r["route_dispatch_ms"] >= 0.0
    assert r["single_thread_tokens_per_s"] > 0.0


def test_kernel_traffic_lookup(tmp_path):
    # a record keyed by another source hash reads as unknown (None), never as a number
    src = tmp_path / "k.cu"
    src.write_text("// not a recorded source\n")
    assert bench.kernel_traffic(str(src), "gate_up", "decode_t1") is None
    assert bench.kernel_traffic(str(src), "gate_up", "no_such_workload") is None
