"""Host-side pieces of bench.py that need no GPU: the oracle timings of the
cpu_baseline object, the DRAM-traffic lookup and the launch count per step."""
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


def test_resident_layers_defeat_l2():
    # decode: enough layers that the others' weights exceed four times the L2
    w = synth.WORKLOADS["decode_t1"]
    n = bench.resident_layers(w, 8)
    per_step = 7 * synth.expert_bytes(w.d, w.f)
    assert (n - 1) * per_step >= 4 * bench.L2_BYTES and n <= 8
    # prefill reads the whole layer every step: two layers suffice; 43 layers stay 43
    assert bench.resident_layers(synth.WORKLOADS["prefill_t4096_uniform"], 8) == 2
    assert bench.resident_layers(synth.WORKLOADS["layers43_t32"], 8) == 43


def test_fp8_peak_choice():
    assert bench.fp8_peak_of({"mxfp8_tflops": 4000.0, "fp8_tensorwise_tflops": 4100.0},
                             1600.0)[0] == 4000.0
    assert bench.fp8_peak_of({"fp8_tensorwise_tflops": 4100.0}, 1600.0)[0] == 4100.0
    peak, src = bench.fp8_peak_of({}, 1600.0)
    assert peak == 3200.0 and "nominal" in src


def test_launches_per_step():
    # the layer kernels a step launches, as the library picks them by batch size
    assert bench.launches_per_step(1, 6, fused=True, batched=False) == 1
    # batched GEMV path: route, dispatch, prepare, gate/up, quant_h, down, combine
    assert bench.launches_per_step(64, 6, fused=False, batched=True) == 7
    assert bench.launches_per_step(32, 6, fused=False, batched=True) == 7
    # tile path below 2048 pairs: route, dispatch, prepare, gate/up, down, combine
    assert bench.launches_per_step(100, 8, fused=False, batched=False) == 6
    # prefill: the dispatch and the prepare step are two kernels each
    assert bench.launches_per_step(4096, 6, fused=False, batched=False) == 8
    assert bench.launches_per_step(512, 6, fused=False, batched=False) == 7
