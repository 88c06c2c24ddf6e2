#!/usr/bin/env python3
"""Benchmark of the routed-expert MoE layer (route -> dispatch -> FP4 expert FFN -> combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole layer over one batch of synthetic tokens, with the
layer's weights resident in HBM.  Default workload: one decode layer, T=1 token,
256 routed experts + 1 shared, top-6, d=4096, f=2048 (FP4 e2m1 weights, e4m3
activations).  The steps rotate over several resident layers, each with its own weights
and tokens, so that a step never finds its weights in L2 from before (inputs larger than
L2).  The K timed steps are captured back to back in one CUDA graph (as a model runs its
layers) and timed with CUDA events; a second figure times each step as its own graph
replay.  Multi-GPU runs are replicas (each rank its own tokens and weights, no collective
on the data path) -> weak scaling.

At one GPU the line also carries a `workloads` record: the batched-decode (T=64, Zipf 1.0),
prefill (T=4096, uniform and Zipf 1.2) and 43-resident-layer (T=1 and T=32, Zipf 1.0)
configurations, each with its step time, the dominant kernel's roofline, the layer-level
fraction and an oracle sample; and `peaks`, the dense FP8 tensor rate measured on this GPU.

Prints one JSON line (rank 0).  `--impl reference` times the oracle (the plain CPU
implementation the tests check against) on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s; decode HBM GB/s and prefill TFLOPS as % of B200 peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
SPEC_HBM_GBS = 8000.0          # B200 HBM3e, spec
SPEC_FP8_TFLOPS = 4500.0       # B200 dense FP8, spec
L2_BYTES = 126 * 2 ** 20
EXTRA_WORKLOADS = ("decode_t64_zipf", "prefill_t4096_uniform", "prefill_t4096_zipf",
                   "layers43_t1", "layers43_t32", "decode_t1_q2")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return j.get("hbm_gbs", FALLBACK_HBM_GBS), j.get("bf16_tflops", FALLBACK_BF16_TFLOPS), \
            j.get("bf16_tflops_sustained", FALLBACK_BF16_TFLOPS), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


# ------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm = [float(r[1]) for r in self.rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            if len(r) >= 9:
                for n, v in zip(names, r[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------ algorithmic work
def layer_work(w, counts: np.ndarray):
    """Algorithmic bytes of the gate/up launch and of the whole FFN, and the flops, for
    the experts that have tokens (the shared expert always does)."""
    d, f, T, k = w.d, w.f, w.T, w.k
    active = int((counts > 0).sum()) + 1
    R = T * k + T
    gu_w = 2 * (f * d // 2 + f * d // 32)            # gate + up codes and scales per expert
    dn_w = d * f // 2 + d * f // 32
    weight_bytes = active * (gu_w + dn_w)
    if w.routed_codec == "q2":  # routed experts 2-bit (codes K/4, scales K/128 per row)
        q2_w = 3 * (f * d // 4 + f * d // 128)
        weight_bytes = (active - 1) * q2_w + gu_w + dn_w
    gu_bytes = active * gu_w + R * d + R * (d // 128) * 4 + R * f + R * (f // 128) * 4
    dn_bytes = active * dn_w + R * f + R * (f // 128) * 4 + R * d * 4
    flops_gu = 2 * 2 * R * d * f
    flops_dn = 2 * R * d * f
    return dict(active=active, gu_bytes=gu_bytes, dn_bytes=dn_bytes, flops_gu=flops_gu,
                flops_dn=flops_dn, weight_bytes=weight_bytes)


def kernel_traffic(kernel_file: str, name: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on this kernel source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as fh:
            j = json.load(fh)
        src = hashlib.sha256(open(kernel_file, "rb").read()).hexdigest()[:16]
        e = j.get(workload, {}).get(name)
        if e and e.get("source_sha") == src:
            return e.get("bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


def max_over_ranks(seconds: float, dist, device) -> float:
    """Largest value over all ranks (the job's time is the slowest rank's time)."""
    if dist is None:
        return seconds
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(w, rank: int) -> int:
    """Each rank of a multi-GPU run serves its own tokens (replicas, weak scaling)."""
    return w.seed(0) + 100000 * rank


def time_graph(g, stream, reps: int) -> list:
    """Durations (ms) of `reps` replays of a CUDA graph, each after a short device sleep so
    that the timed region does not start before the host has queued the replay."""
    out = []
    with torch.cuda.stream(stream):
        for _ in range(reps):
            torch.cuda._sleep(100000)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            out.append((e0, e1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in out]


# ------------------------------------------------------------------------ measured peaks
def measure_fp8_peak(dev) -> dict:
    """Dense FP8 (e4m3 x e4m3 -> bf16) GEMM rate of this GPU through torch._scaled_mm on
    8192^3: with one scale per tensor, and block-scaled (one e8m0 scale per 32 elements
    along K, the MX format) where the build supports it.  Timed alone (burst) with CUDA
    events, median of 20 after 5 warm-ups."""
    M = N = K = 8192
    res = {"how": "torch._scaled_mm e4m3 x e4m3 -> bf16, 8192^3, CUDA events, median of 20"}
    a = torch.randn(M, K, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(N, K, device=dev).to(torch.float8_e4m3fn).t()
    one = torch.tensor(1.0, device=dev)

    def timed(fn):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(20):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            ts.append((e0, e1))
        torch.cuda.synchronize()
        ms = statistics.median(x.elapsed_time(y) for x, y in ts)
        return 2.0 * M * N * K / (ms * 1e-3) / 1e12

    try:
        res["fp8_tensorwise_tflops"] = timed(
            lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16))
    except Exception as e:  # noqa: BLE001 - recorded, not fatal
        res["fp8_tensorwise_error"] = f"{type(e).__name__}: {str(e)[:160]}"
    try:
        e8 = torch.float8_e8m0fnu
        sa = torch.full((M, K // 32), 127, dtype=torch.uint8, device=dev).view(e8)
        sb = torch.full((N, K // 32), 127, dtype=torch.uint8, device=dev).view(e8)
        res["mxfp8_tflops"] = timed(
            lambda: torch._scaled_mm(a, b, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16))
    except Exception as e:  # noqa: BLE001
        res["mxfp8_error"] = f"{type(e).__name__}: {str(e)[:160]}"
    del a, b
    torch.cuda.empty_cache()
    return res


def fp8_peak_of(peaks: dict, bf16_peak: float):
    if peaks.get("mxfp8_tflops"):
        return peaks["mxfp8_tflops"], "measured dense MX block-scaled FP8 (torch._scaled_mm)"
    if peaks.get("fp8_tensorwise_tflops"):
        return peaks["fp8_tensorwise_tflops"], "measured dense FP8, one scale per tensor " \
                                               "(torch._scaled_mm)"
    return 2.0 * bf16_peak, "2 x bf16 burst (nominal fp8/bf16 ratio; FP8 not measurable)"


# ------------------------------------------------------------------------ CPU oracle leg
def host_expert_for(w, layer_seed: int, e: int):
    """Host copy of expert e as the oracle takes it (2-bit routed experts tagged with
    their codec; the shared expert, index E, is FP4)."""
    import oracle
    if w.routed_codec == "q2" and e < w.E:
        he = synth.host_expert_q2(layer_seed, 0, e, w.d, w.f)
        ex = type("Q2Expert", (), {})()
        ex.__dict__.update(he.__dict__)
        ex.codec = oracle.Q2
        return ex
    return synth.host_expert(layer_seed, 0, e, w.d, w.f)


def oracle_sample(w, x, scores, seconds: float, layer_seed: int):
    """Time the oracle on whole tokens of this workload for about `seconds` seconds.
    Returns (tokens/s, cores, description)."""
    import oracle
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    idx, gw = oracle.route_topk(scores.numpy(), w.k)
    n_tok, cache, elapsed = 0, {}, 0.0
    while elapsed < seconds:
        t = n_tok % w.T
        need = set(idx[t].tolist()) | {w.E}
        for e in need:  # weight generation is input preparation, not timed
            if e not in cache:
                cache[e] = host_expert_for(w, layer_seed, e)
        ta = time.perf_counter()
        oracle.moe_tokens(x, w.E, w.k, w.d, w.f, {e: cache[e] for e in need}, idx, gw, [t])
        elapsed += time.perf_counter() - ta
        n_tok += 1
    return n_tok / elapsed, cores, \
        f"{n_tok} whole tokens of this workload (quantise, {w.k} routed + 1 shared expert " \
        f"FFN, combine), {elapsed:.1f} s of oracle time on {cores} threads"


def oracle_extras(w, x, scores, layer_seed: int) -> dict:
    """The oracle's routing + dispatch time for the whole batch, and one token's time on a
    single thread (weights prepared beforehand, untimed)."""
    import oracle
    s_np = scores.numpy()
    ta = time.perf_counter()
    idx, gw = oracle.route_topk(s_np, w.k)
    oracle.dispatch(idx, w.E)
    route_s = time.perf_counter() - ta
    need = set(idx[0].tolist()) | {w.E}
    experts = {e: host_expert_for(w, layer_seed, e) for e in need}
    cores = os.cpu_count() or 1
    oracle.set_threads(1)
    try:
        ta = time.perf_counter()
        oracle.moe_tokens(x, w.E, w.k, w.d, w.f, experts, idx, gw, [0])
        one_s = time.perf_counter() - ta
    finally:
        oracle.set_threads(cores)
    return {"route_dispatch_ms": 1000.0 * route_s,
            "single_thread_tokens_per_s": 1.0 / one_s}


def cpu_baseline(w, x, scores, seconds, extras=False):
    import oracle
    oracle.build()
    rate, cores, desc = oracle_sample(w, x, scores, seconds, w.seed(0))
    cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
    if extras:
        cpu.update(oracle_extras(w, x, scores, w.seed(0)))
    return cpu


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x, scores = synth.gen_layer_inputs(w, 0)
    import oracle
    oracle.build()
    per_step = args.ref_seconds if args.ref_seconds else \
        max(1.0, min(30.0, 60.0 / max(args.steps + args.warmup, 1)))
    for _ in range(args.warmup):
        oracle_sample(w, x, scores, 0.2, w.seed(0))
    times = []
    tok = 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        rate, cores, desc = oracle_sample(w, x, scores, per_step, w.seed(0))
        times.append(time.perf_counter() - t0)
        tok += rate * times[-1]
    value = tok / sum(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * w.T / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "T": w.T, "E": w.E, "k": w.k, "d": w.d, "f": w.f,
                   "routing": w.routing},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------ GPU leg
class Layers:
    """L resident layers of a workload on one device, each with its own weights and tokens."""

    def __init__(self, bm, w, n_layers, rank, dev):
        T, k, E, d, f = w.T, w.k, w.E, w.d, w.f
        self.w = w
        self.items = []
        for l in range(n_layers):
            seed = replica_seed(w, rank) + l if w.layers == 1 else w.seed(l)
            if rank == 0 or w.layers > 1:
                x_cpu, s_cpu = synth.gen_layer_inputs(w, l)
            else:
                x_cpu = synth.gen_x(T, d, seed)
                s_cpu = synth.gen_scores_uniform(T, E, seed) if w.routing == "uniform" else \
                    synth.gen_scores_zipf(T, E, w.zipf_s, seed)
            W = bm.LayerWeights.from_dict(synth.device_layer_weights(w.seed(l), l, E, d, f))
            Q = bm.Q2Experts.from_dict(synth.device_layer_weights_q2(w.seed(l), l, E, d, f)) \
                if w.routed_codec == "q2" else None
            self.items.append(dict(x_cpu=x_cpu, s_cpu=s_cpu, W=W, Q=Q, x=x_cpu.to(dev),
                                   scores=s_cpu.to(dev)))
        self.ws = bm.alloc_workspace(T, k, E, d, f, dev)
        i32, f32 = torch.int32, torch.float32
        self.outs = {"idx": torch.empty((T, k), dtype=i32, device=dev),
                     "w": torch.empty((T, k), dtype=f32, device=dev),
                     "counts": torch.empty((E,), dtype=i32, device=dev),
                     "offsets": torch.empty((E + 1,), dtype=i32, device=dev),
                     "perm": torch.empty((max(T * k, 1),), dtype=i32, device=dev),
                     "pos": torch.empty((max(T * k, 1),), dtype=i32, device=dev),
                     "y": torch.empty((max(T * k, 1), d), dtype=f32, device=dev),
                     "y_shared": torch.empty((T, d), dtype=f32, device=dev),
                     "out": torch.empty((T, d), dtype=f32, device=dev)}


def launches_per_step(T: int, k: int, fused: bool, batched: bool) -> int:
    """This library's kernels in one layer step: one at T = 1 (the fused layer kernel);
    otherwise route, gate/up, down and combine, the dispatch (two kernels from 8192 pairs),
    and the prepare step (two kernels on the tile path from 2048 pairs: the inverse
    permutation and the per-token quantisation) or, on the batched path, prepare and
    quant_h."""
    if fused:
        return 1
    return 4 + (2 if T * k >= 8192 else 1) + (2 if batched or T * k >= 2048 else 1)


def resident_layers(w, max_layers):
    """Layers to rotate through so that a step's weights have been evicted from L2 by the
    other layers' since their last use (four times the L2 in between)."""
    if w.layers > 1:
        return w.layers
    per_expert = synth.expert_bytes(w.d, w.f)
    routed = synth.q2_expert_bytes(w.d, w.f) if w.routed_codec == "q2" else per_expert
    step_bytes = min(w.E, w.T * w.k) * routed + per_expert
    return max(min(2, max_layers), min(max_layers, -(-4 * L2_BYTES // step_bytes) + 1))


def measure(bm, w, args, dev, stream, rank, dist, steps, warmup, peaks, cpu_seconds,
            headline=False):
    """Time one workload; returns the record (and the layers, for the e2e leg)."""
    T, k, E, d, f = w.T, w.k, w.E, w.d, w.f
    n_layers = resident_layers(w, args.max_layers)
    if w.layers > 1:
        steps = w.layers * max(1, steps // w.layers)  # whole passes over the resident layers
    Ls = Layers(bm, w, n_layers, rank, dev)

    # one step = the whole layer in one call (moe_forward): one kernel for a single token,
    # otherwise route, dispatch, prepare, gate/up, down and combine back to back
    fused = T == 1 and d % 512 == 0 and f % 512 == 0
    batched = 2 <= T <= 64 and d % 512 == 0 and f % 512 == 0  # the batched GEMV path
    q2 = w.routed_codec == "q2"

    def step(L):
        if q2:
            return bm.forward_q2(L["x"], L["scores"], k, L["W"], L["Q"], Ls.ws, stream,
                                 outs=Ls.outs)["counts"]
        return bm.forward(L["x"], L["scores"], k, L["W"], Ls.ws, stream, outs=Ls.outs)["counts"]

    # one eager pass per layer (checks the status word and gives the routing counts)
    works = []
    for L in Ls.items:
        with torch.cuda.stream(stream):
            counts = step(L)
        bm.sync_status(stream)
        works.append(layer_work(w, counts.cpu().numpy()))
    work = {key: sum(wk[key] for wk in works) / len(works) for key in works[0]}

    # the K timed steps back to back in one graph (step i runs layer i % L), a graph of the
    # warm-up steps, and one graph per layer for the isolated per-step figure
    def chain(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                step(Ls.items[i % n_layers])
        return g

    g_warm, g_timed = chain(warmup), chain(steps)
    g_one = []
    for L in Ls.items[:min(n_layers, 8)]:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(L)
        g_one.append(g)

    # the dominant kernel's own duration: graph A runs route, dispatch, prepare and gate/up
    # for every layer in turn, graph B the same without gate/up; gate/up per launch is
    # (A - B) / layers.  Launch latencies cancel, and every gate/up meets its weights cold.
    def pre(L):
        idx, _ = bm.route_topk(L["scores"], k, stream)
        _, offsets, perm, _ = bm.dispatch(idx, E, stream)
        bm.ffn_prepare(L["x"], k, L["W"], offsets, perm, Ls.ws, stream)

    g_a, g_b = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    if not fused:
        with torch.cuda.graph(g_a, stream=stream):
            for L in Ls.items:
                pre(L)
                bm.ffn_gate_up(T, k, L["W"], Ls.ws, stream)
        with torch.cuda.graph(g_b, stream=stream):
            for L in Ls.items:
                pre(L)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        g_warm.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()

    clocks = None
    if headline:
        clocks = ClockSampler(int(str(dev).split(":")[-1]) if ":" in str(dev) else 0)
        clocks.start()
        time.sleep(0.3)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(100000)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g_timed.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    timed_ms = e0.elapsed_time(e1)
    one_ms = []
    for i in range(max(len(g_one), 10)):
        one_ms += time_graph(g_one[i % len(g_one)], stream, 1)
    ab = {"a": [], "b": []}
    if not fused:
        for _ in range(max(7, min(15, steps))):
            ab["a"] += time_graph(g_a, stream, 1)
            ab["b"] += time_graph(g_b, stream, 1)
    clk = clocks.stop() if clocks is not None else None
    total_s = max_over_ranks(timed_ms / 1000.0, dist, dev)
    world = dist.get_world_size() if dist is not None else 1
    layer_s = total_s / steps
    is_prefill = T > 256
    if fused:
        # the dominant kernel is the step itself: K launches back to back in one graph
        gu_s = timed_ms / 1000.0 / steps
        kernel_file = os.path.join(ROOT, "bit_moe_routed_b200", "csrc", "decode.cu")
        kernel_name = ("decode_kernel: the whole layer in one cooperative kernel (routing, "
                       "dispatch, quantisation, FP4 GEMVs with in-register e2m1 decode and "
                       "mma.sync, combine)")
        if not q2 and bm.forward_path(1, k, Ls.items[0]["W"]) == bm.PATH_SINGLE_TC:
            kernel_file = os.path.join(ROOT, "bit_moe_routed_b200", "csrc", "decode_tc.cu")
            kernel_name = ("decode_tc_kernel: the whole layer in one cooperative kernel "
                           "(routing, dispatch, quantisation, tcgen05 block-scaled FP4 x e4m3 "
                           "MMAs on TMA-unpacked codes against block-diagonal token tiles, "
                           "combine)")
        if q2:
            kernel_name = ("decode_kernel, Q2 form: the whole layer in one cooperative kernel, "
                           "2-bit routed experts (byte-permute decode to e4m3, mma.sync e4m3) "
                           "and the FP4 shared expert")
        traffic = kernel_traffic(kernel_file, "layer_tc" if kernel_file.endswith("decode_tc.cu")
                                 else "layer", w.name)
        io = 4 * E + 2 * d + 4 * d * (k + 2)  # scores, x; y_routed, y_shared and out
        work["gu_bytes"] = work["weight_bytes"] + io
    else:
        gu_s = (statistics.median(ab["a"]) - statistics.median(ab["b"])) / n_layers / 1000.0
        if batched:
            kernel_file = os.path.join(ROOT, "bit_moe_routed_b200", "csrc", "bgemv.cu")
            kernel_name = ("bgemv gate/up + SwiGLU (batched FP4 GEMV: packed codes in shared "
                           "memory, in-register e2m1 decode, tokens in mma.sync N columns)")
        else:
            kernel_file = os.path.join(ROOT, "bit_moe_routed_b200", "csrc", "ffn.cu")
            kernel_name = "ffn gate/up (tcgen05 kind::mxf8f6f4)"
        traffic = kernel_traffic(kernel_file, "gate_up", w.name)
    hbm_peak, fp8_peak, fp8_src, peak_kind = peaks
    if is_prefill:
        achieved = work["flops_gu"] / gu_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                "frac": achieved / fp8_peak, "traffic": traffic, "kernel": kernel_name,
                "peak_source": fp8_src}
        layer_tf = (work["flops_gu"] + work["flops_dn"]) / layer_s / 1e12
        layer = {"tflops": layer_tf, "frac_of_measured_fp8": layer_tf / fp8_peak,
                 "frac_of_spec_fp8_4500": layer_tf / SPEC_FP8_TFLOPS,
                 "weight_gb_per_s": work["weight_bytes"] / layer_s / 1e9}
    else:
        achieved = work["gu_bytes"] / gu_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic, "kernel": kernel_name,
                "peak_source": f"{peak_kind} HBM copy"}
        gbs = work["weight_bytes"] / layer_s / 1e9
        layer = {"weight_gb_per_s": gbs, "weight_bytes": work["weight_bytes"],
                 "frac_of_measured_hbm": gbs / hbm_peak, "frac_of_spec_hbm_8tbs": gbs / SPEC_HBM_GBS,
                 "tflops": (work["flops_gu"] + work["flops_dn"]) / layer_s / 1e12}
    roof["avg_launch_us"] = gu_s * 1e6
    roof["algorithmic_per_launch"] = work["flops_gu"] if is_prefill else work["gu_bytes"]
    rec = {
        "fused": fused, "launches_per_step": launches_per_step(T, k, fused, batched),
        "value": world * T * steps / total_s, "unit": "tokens/s", "steps": steps,
        "ms_per_step": 1000.0 * layer_s,
        "ms_per_step_isolated": statistics.median(one_ms),
        "config": {"workload": w.name, "T": T, "E": E, "k": k, "d": d, "f": f,
                   "routing": w.routing, "zipf_s": w.zipf_s if w.routing == "zipf" else None,
                   "active_experts": work["active"], "resident_layers": n_layers},
        "layer": layer, "roofline": roof,
    }
    if clk is not None:
        rec["clocks"] = clk
    if rank == 0 and world == 1 and cpu_seconds > 0:
        x_cpu, s_cpu = Ls.items[0]["x_cpu"], Ls.items[0]["s_cpu"]
        rec["cpu_baseline"] = cpu_baseline(w, x_cpu, s_cpu, cpu_seconds, extras=T <= 64 and headline)
    del g_warm, g_timed, g_one, g_a, g_b
    return rec, Ls


def measure_shared_fp8(bm, dev, stream, T: int, hbm_peak: float, peak_kind: str,
                       steps: int = 20) -> dict:
    """The FP8-weight shared expert (moe_shared_expert_fp8) at d = 4096, f = 2048 for T
    tokens: `steps` calls back to back in one CUDA graph, each on its own copy of the
    weights (enough copies that a copy's 25 MB were evicted from L2 since its last use)."""
    d, f = 4096, 2048
    wbytes = synth.fp8_expert_bytes(d, f)
    n = max(2, -(-4 * L2_BYTES // wbytes) + 1)
    experts = [bm.Fp8Expert.from_dict(synth.device_expert_fp8(2000 + i, 0, d, f)) for i in range(n)]
    x = synth.gen_x(T, d, seed=77).to(dev)
    ws = torch.empty(int(bm.lib().moe_shared_expert_fp8_workspace_size(T, d, f)), dtype=torch.uint8,
                     device=dev)
    y = torch.empty((T, d), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        for i in range(n):  # eager pass over every copy (checks the status word)
            bm.shared_expert_fp8(x, experts[i], ws=ws, stream=stream, out=y)
    bm.sync_status(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            bm.shared_expert_fp8(x, experts[i % n], ws=ws, stream=stream, out=y)
    time_graph(g, stream, 3)
    ms = statistics.median(time_graph(g, stream, 5)) / steps
    s = ms / 1000.0
    gbs = wbytes / s / 1e9
    del g
    return {"T": T, "d": d, "f": f, "ms_per_step": ms, "steps": steps, "resident_copies": n,
            "value": T / s, "unit": "tokens/s", "launches_per_step": 4,
            "weight_bytes": wbytes, "weight_gb_per_s": gbs, "frac_of_measured_hbm": gbs / hbm_peak,
            "peak_source": f"{peak_kind} HBM copy",
            "kernels": "quant_rows (x -> e4m3), fp8_gemm gate+up -> h, quant_h, fp8_gemm down "
                       "(mma.sync e4m3 on the codes, cp.async weight tiles)"}


def measure_streamed(bm, dev, stream, S: int = 64, steps: int = 64, zipf_s: float = 1.0) -> dict:
    """Decode T = 1 with the 256 routed experts in pinned host memory and an HBM cache of S
    slots (moe_forward_streamed): `steps` tokens with Zipf(zipf_s) routing, one CUDA graph,
    after as many untimed tokens to fill the cache.  Also the H2D copy rate of pinned host
    memory (the bound of the fetches)."""
    w = synth.WORKLOADS["decode_t1"]
    E, k, d, f = w.E, w.k, w.d, w.f
    W = bm.LayerWeights.from_dict(synth.device_layer_weights(w.seed(0), 0, E, d, f))
    host = bm.HostExperts.from_layer(W)
    cache = bm.ExpertCache(E, S, d, f, W)
    del W
    torch.cuda.empty_cache()
    ws = bm.alloc_workspace(1, k, E, d, f, dev)
    xs = [synth.gen_x(1, d, seed=9000 + i).to(dev) for i in range(2 * steps)]
    ss = [synth.gen_scores_zipf(1, E, zipf_s, seed=9000 + i).to(dev) for i in range(2 * steps)]
    outs = None
    with torch.cuda.stream(stream):
        for i in range(steps):  # untimed: fill the cache
            outs = bm.forward_streamed(xs[i], ss[i], k, host, cache, ws, stream, outs=outs)
    bm.sync_status(stream)
    st0 = cache.stats.cpu().tolist()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps, 2 * steps):
            bm.forward_streamed(xs[i], ss[i], k, host, cache, ws, stream, outs=outs)
    ms = time_graph(g, stream, 1)[0]
    bm.sync_status(stream)
    st1 = cache.stats.cpu().tolist()
    hits, misses = st1[0] - st0[0], st1[1] - st0[1]
    per_expert = synth.expert_bytes(d, f)
    # pinned host -> device copy rate, 1 GiB (the PCIe bound of the fetches)
    hb = torch.empty(1 << 30, dtype=torch.uint8, pin_memory=True)
    db = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        db.copy_(hb, non_blocking=True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        db.copy_(hb, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    h2d = (1 << 30) / (e0.elapsed_time(e1) / 1000.0) / 1e9
    s_step = ms / 1000.0 / steps
    fetched = misses * per_expert / steps
    del g, hb, db, host, cache
    torch.cuda.empty_cache()
    return {"T": 1, "E": E, "k": k, "d": d, "f": f, "slots": S, "zipf_s": zipf_s,
            "steps": steps, "ms_per_step": ms / steps, "value": 1.0 / s_step,
            "unit": "tokens/s", "hit_rate": hits / max(hits + misses, 1),
            "fetched_bytes_per_step": fetched, "fetch_gb_per_s": fetched / s_step / 1e9,
            "h2d_copy_gb_per_s": h2d, "frac_of_h2d_copy": fetched / s_step / 1e9 / h2d,
            "launches_per_step": 4,
            "how": "route, cache (LRU), fetch (host-mapped reads) and the single-token layer "
                   "kernel per token, in one CUDA graph; the H2D rate is a 1 GiB pinned copy"}


def e2e(bm, Ls, args, dev, stream, dist, world):
    """The same metric through the public API with host buffers: each step copies x and the
    scores from pinned host memory, runs the four calls and copies the output back, then
    synchronises (a decode loop needs each output before its next input).  Measured as one
    CUDA graph per layer, and eagerly (the four calls issued from Python each step)."""
    w = Ls.w
    T, k, d, E = w.T, w.k, w.d, w.E
    for L in Ls.items:
        L["x_h"] = L["x_cpu"].pin_memory()
        L["s_h"] = L["s_cpu"].pin_memory()
    out_h = torch.empty((T, d), dtype=torch.float32).pin_memory()

    def body(L):
        L["x"].copy_(L["x_h"], non_blocking=True)
        L["scores"].copy_(L["s_h"], non_blocking=True)
        r = bm.forward(L["x"], L["scores"], k, L["W"], Ls.ws, stream)
        out_h.copy_(r["out"], non_blocking=True)

    g_e2e = []
    for L in Ls.items:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            body(L)
        g_e2e.append(g)
    torch.cuda.synchronize()
    res = {}
    for mode in ("graph", "eager"):
        ms = []
        for i in range(args.warmup + args.steps):
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                a.record(stream)
                if mode == "graph":
                    g_e2e[i % len(g_e2e)].replay()
                else:
                    body(Ls.items[i % len(Ls.items)])
                b.record(stream)
            b.synchronize()
            if i >= args.warmup:
                ms.append(a.elapsed_time(b))
        s = max_over_ranks(sum(ms) / 1000.0, dist, dev)
        res[mode] = world * T * args.steps / s
    bm.sync_status(stream)
    del g_e2e
    return {"value": res["graph"], "unit": "tokens/s",
            "h2d_bytes_per_step": T * d * 2 + T * E * 4, "d2h_bytes_per_step": T * d * 4,
            "how": "per layer one CUDA graph of the pinned H2D copies of x and scores, the four "
                   "calls and the D2H copy of out; synchronised every step",
            "eager_value": res["eager"],
            "eager_how": "the same copies and the four calls issued from Python (ctypes) every "
                         "step, no graph: includes the host's launch costs"}


def run_gpu(args, w):
    import bit_moe_routed_b200 as bm
    bm.set_decode_engine(args.decode_engine)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(dev)
    hbm_peak, bf16_peak, bf16_sus, peak_kind = load_peaks()
    fp8 = measure_fp8_peak(dev) if world == 1 and not args.no_workloads else {}
    fp8_peak, fp8_src = fp8_peak_of(fp8, bf16_peak)
    peaks = (hbm_peak, fp8_peak, fp8_src, peak_kind)

    rec, Ls = measure(bm, w, args, dev, stream, rank, dist, args.steps, args.warmup, peaks,
                         0 if args.no_cpu_baseline else args.cpu_seconds, headline=True)
    e2e_rec = e2e(bm, Ls, args, dev, stream, dist, world)
    del Ls
    torch.cuda.empty_cache()

    workloads = {}
    if world == 1 and not args.no_workloads:
        names = EXTRA_WORKLOADS if args.workloads == "all" else \
            [n for n in args.workloads.split(",") if n]
        for name in names:
            if name == w.name or name not in synth.WORKLOADS:
                continue
            wl = synth.WORKLOADS[name]
            need = (wl.layers if wl.layers > 1 else 2) * synth.expert_bytes(wl.d, wl.f) * (wl.E + 1)
            free, _ = torch.cuda.mem_get_info(dev)
            if free < need + (6 << 30):
                workloads[name] = {"skipped": f"needs {need / 1e9:.1f} GB, {free / 1e9:.1f} GB free"}
                continue
            r, Lw = measure(bm, wl, args, dev, stream, rank, dist,
                            args.extra_steps, 3, peaks, args.extra_cpu_seconds)
            workloads[name] = r
            del Lw
            import gc
            gc.collect()
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        if args.workloads == "all" or "streamed" in args.workloads:
            workloads["streamed_t1"] = measure_streamed(bm, dev, stream)
            torch.cuda.empty_cache()
        if args.workloads == "all" or "shared_fp8" in args.workloads:
            for Tf in (1, 64):  # NEXT-3: the FP8-weight shared expert on fp8_gemm
                workloads[f"shared_fp8_t{Tf}"] = measure_shared_fp8(bm, dev, stream, Tf, hbm_peak,
                                                                     peak_kind)
            torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": rec["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e2m1 x e4m3 -> f32", "data": "synthetic (seeded weights and tokens)",
            "config": dict(rec["config"], **{
                "l2": f"not flushed: step i runs layer i % {rec['config']['resident_layers']}, "
                      "each with its own weights, so a step's weights were evicted by the other "
                      "layers since their last use (inputs larger than L2)",
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "launch": "the K timed steps captured back to back in one CUDA graph"}),
            "ms_per_step_isolated": rec["ms_per_step_isolated"],
            "layer": rec["layer"],
            "roofline": rec["roofline"],
            "cpu_baseline": rec.get("cpu_baseline"),
            "e2e": e2e_rec,
            "gpu_launches": rec["launches_per_step"] * args.steps,
            "clocks": rec.get("clocks"),
            "peaks": dict(fp8, hbm_gbs=hbm_peak, hbm_source=peak_kind,
                          fp8_used_tflops=fp8_peak, fp8_used_source=fp8_src,
                          bf16_burst_tflops=bf16_peak),
            "workloads": workloads,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_t1", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="bitmoe", choices=["bitmoe", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--max-layers", type=int, default=8,
                    help="most layers kept resident to rotate through (defeats L2 reuse)")
    ap.add_argument("--workloads", default="all",
                    help="extra workloads to record at one GPU: 'all' or a comma list")
    ap.add_argument("--no-workloads", action="store_true", help="headline workload only")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--extra-cpu-seconds", type=float, default=4.0)
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="oracle seconds per step of the reference arm (default: fit ~1 min)")
    ap.add_argument("--decode-engine", type=int, default=0, choices=[0, 1],
                    help="single-token layer kernel of moe_forward: 0 CUDA cores (default), "
                         "1 tensor cores")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        synth.build()
        run_gpu(args, w)


if __name__ == "__main__":
    main()
