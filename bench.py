#!/usr/bin/env python3
"""Benchmark of the routed-expert MoE layer (route -> dispatch -> FP4 expert FFN -> combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole layer over one batch of synthetic tokens, with the
layer's weights resident in HBM.  Default workload: one decode layer, T=1 token,
256 routed experts + 1 shared, top-6, d=4096, f=2048 (FP4 e2m1 weights, e4m3
activations).  Each step is one layer; the steps rotate over several resident layers,
each with its own weights and tokens, so that a step never finds its weights in L2 from
before (inputs larger than L2).  Each layer's step is captured once in a CUDA graph and
replayed.  Multi-GPU runs are replicas
(each rank its own tokens and weights, no collective on the data path) -> weak scaling.

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
    gu_bytes = active * gu_w + R * d + R * (d // 128) * 4 + R * f + R * (f // 128) * 4
    dn_bytes = active * dn_w + R * f + R * (f // 128) * 4 + R * d * 4
    flops_gu = 2 * 2 * R * d * f
    flops_dn = 2 * R * d * f
    return dict(active=active, gu_bytes=gu_bytes, dn_bytes=dn_bytes, flops_gu=flops_gu,
                flops_dn=flops_dn, weight_bytes=active * (gu_w + dn_w))


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


# ------------------------------------------------------------------------ CPU oracle leg
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
                cache[e] = synth.host_expert(layer_seed, 0, e, w.d, w.f)
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
    experts = {e: synth.host_expert(layer_seed, 0, e, w.d, w.f) for e in need}
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
def run_gpu(args, w):
    import bit_moe_routed_b200 as bm
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
    hbm_peak, bf16_peak, bf16_sus, peak_kind = load_peaks()

    # Working set: L layers resident in HBM, each with its own weights and tokens; step i
    # runs layer i % L.  L is chosen so the other L-1 layers' weights exceed four times
    # the L2, so a step's weights are never still in L2 from its previous use (read-only
    # weights: no dirty lines to write back, unlike a write-flush).
    T, k, E, d, f = w.T, w.k, w.E, w.d, w.f
    per_expert = synth.expert_bytes(d, f)
    est_active = min(E, T * k) + 1
    step_bytes = est_active * per_expert
    L2_BYTES = 126 * 2 ** 20
    n_layers = max(min(2, args.max_layers), min(args.max_layers, -(-4 * L2_BYTES // step_bytes) + 1))
    layers = []
    for l in range(n_layers):
        seed = replica_seed(w, rank) + l
        if rank == 0:
            x_cpu, s_cpu = synth.gen_layer_inputs(w, l)
        else:
            x_cpu = synth.gen_x(T, d, seed)
            s_cpu = synth.gen_scores_uniform(T, E, seed) if w.routing == "uniform" else \
                synth.gen_scores_zipf(T, E, w.zipf_s, seed)
        W = bm.LayerWeights.from_dict(synth.device_layer_weights(w.seed(l), l, E, d, f))
        layers.append(dict(x_cpu=x_cpu, s_cpu=s_cpu, W=W, x=x_cpu.to(dev), scores=s_cpu.to(dev)))
    ws = bm.alloc_workspace(T, k, E, d, f, dev)
    y = torch.empty((T * k, d), dtype=torch.float32, device=dev)
    ysh = torch.empty((T, d), dtype=torch.float32, device=dev)
    out = torch.empty((T, d), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)

    def step(L):
        # route -> dispatch -> FFN (prepare | gate/up | down) -> combine
        idx, gw = bm.route_topk(L["scores"], k, stream)
        counts, offsets, perm, pos = bm.dispatch(idx, E, stream)
        bm.expert_ffn(L["x"], k, L["W"], offsets, perm, ws, out=(y, ysh), stream=stream)
        bm.combine(y, ysh, gw, pos, out, stream)
        return counts

    # one eager pass per layer (checks the status word), then one graph per layer of the
    # whole step, and one of the gate/up kernel alone (after its own prepare) per layer
    works = []
    for L in layers:
        with torch.cuda.stream(stream):
            counts = step(L)
        bm.sync_status(stream)
        works.append(layer_work(w, counts.cpu().numpy()))
    work = works[0]
    g_step = []
    for L in layers:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(L)
        g_step.append(g)

    # The dominant kernel's own duration: graph A runs route, dispatch, prepare and gate/up
    # for every layer in turn, graph B the same without gate/up; gate/up per launch is
    # (A - B) / layers.  Launch latencies cancel, and every gate/up meets its weights cold.
    def pre(L):
        idx, _ = bm.route_topk(L["scores"], k, stream)
        _, offsets, perm, _ = bm.dispatch(idx, E, stream)
        bm.ffn_prepare(L["x"], k, L["W"], offsets, perm, ws, stream)

    g_a, g_b = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_a, stream=stream):
        for L in layers:
            pre(L)
            bm.ffn_gate_up(T, k, L["W"], ws, stream)
    with torch.cuda.graph(g_b, stream=stream):
        for L in layers:
            pre(L)
    torch.cuda.synchronize()

    for i in range(args.warmup):
        with torch.cuda.stream(stream):
            g_step[i % n_layers].replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            starts[i].record(stream)
            g_step[i % n_layers].replay()
            ends[i].record(stream)
        # the dominant kernel: graphs A and B alternately (a sleep first, so that the timed
        # region does not start before the host has queued the graph)
        ab = {"a": [], "b": []}
        for i in range(max(15, args.steps)):
            for name, gr in (("a", g_a), ("b", g_b)):
                torch.cuda._sleep(100000)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                gr.replay()
                e1.record(stream)
                ab[name].append((e0, e1))
    torch.cuda.synchronize()
    clk = clocks.stop()
    ta = statistics.median(e0.elapsed_time(e1) for e0, e1 in ab["a"])
    tb = statistics.median(e0.elapsed_time(e1) for e0, e1 in ab["b"])
    gu_ms = [(ta - tb) / n_layers]
    step_ms = [starts[i].elapsed_time(ends[i]) for i in range(args.steps)]
    total_s = max_over_ranks(sum(step_ms) / 1000.0, dist, dev)
    if dist is not None:
        dist.barrier()
    value = world * T * args.steps / total_s

    # e2e through the public API with host buffers: per layer one CUDA graph of the pinned
    # H2D copies of x and scores, the four calls and the D2H copy of the layer output,
    # replayed for step i (layer i % L) and synchronised before the next step, as a decode
    # loop that needs each output before its next input would run it
    for L in layers:
        L["x_h"] = L["x_cpu"].pin_memory()
        L["s_h"] = L["s_cpu"].pin_memory()
    out_h = torch.empty((T, d), dtype=torch.float32).pin_memory()
    g_e2e = []
    for L in layers:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            L["x"].copy_(L["x_h"], non_blocking=True)
            L["scores"].copy_(L["s_h"], non_blocking=True)
            r = bm.forward(L["x"], L["scores"], k, L["W"], ws, stream)
            out_h.copy_(r["out"], non_blocking=True)
        g_e2e.append(g)
    torch.cuda.synchronize()
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g_e2e[i % n_layers].replay()
            b.record(stream)
        b.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e_s = max_over_ranks(sum(e2e_ms) / 1000.0, dist, dev)
    e2e_value = world * T * args.steps / e2e_s
    bm.sync_status(stream)
    x_cpu, s_cpu = layers[0]["x_cpu"], layers[0]["s_cpu"]

    gu_avg_s = statistics.mean(gu_ms) / 1000.0
    # per-launch algorithmic work averaged over the rotated layers
    work = dict(work)
    for key in ("gu_bytes", "dn_bytes", "flops_gu", "flops_dn", "weight_bytes", "active"):
        work[key] = sum(wk[key] for wk in works) / len(works)
    is_prefill = T > 256
    # single-token batches run the FP4 GEMV kernels (the library's default switch)
    gemv = T == 1 and d % 512 == 0 and f % 512 == 0
    kernel_file = os.path.join(ROOT, "bit_moe_routed_b200", "csrc", "gemv.cu" if gemv else "ffn.cu")
    kernel_name = ("ffn gate/up (FP4 GEMV: TMA-staged rows, in-register e2m1 decode, "
                   "mma.sync f16 -> fp32)") if gemv else "ffn gate/up (tcgen05 kind::mxf8f6f4)"
    traffic = kernel_traffic(kernel_file, "gate_up", w.name)
    if is_prefill:
        fp8_peak = bf16_peak * 2.0  # dense FP8 = 2x dense BF16 (nominal 4.5 / 2.25 PF)
        achieved = work["flops_gu"] / gu_avg_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                "frac": achieved / fp8_peak, "traffic": traffic,
                "kernel": "ffn gate/up (tcgen05 kind::mxf8f6f4)",
                "peak_source": f"{peak_kind} bf16 burst x 2 (nominal fp8/bf16 ratio)"}
    else:
        achieved = work["gu_bytes"] / gu_avg_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic,
                "kernel": kernel_name,
                "peak_source": f"{peak_kind} HBM copy"}
    roof["avg_launch_us"] = gu_avg_s * 1e6
    roof["algorithmic_per_launch"] = work["gu_bytes"] if not is_prefill else work["flops_gu"]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        rate, cores, desc = oracle_sample(w, x_cpu, s_cpu, args.cpu_seconds, w.seed(0))
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
        if T <= 64:  # one token single-threaded is seconds at these sizes
            cpu.update(oracle_extras(w, x_cpu, s_cpu, w.seed(0)))

    if rank == 0:
        layer_s = total_s / args.steps
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * layer_s,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e2m1 x e4m3 -> f32", "data": "synthetic (seeded weights and tokens)",
            "config": {"workload": w.name, "T": T, "E": E, "k": k, "d": d, "f": f,
                       "routing": w.routing, "active_experts": work["active"],
                       "l2": f"not flushed: step i runs layer i % {n_layers}, each with its own "
                             f"weights ({n_layers * 257 * per_expert / 1e9:.1f} GB resident), so a "
                             "step's weights were evicted by the other layers since their last use",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "launch": "one CUDA graph of the 6 kernels per layer"},
            "layer": {"weight_gb_per_s": work["weight_bytes"] / layer_s / 1e9,
                      "weight_bytes": work["weight_bytes"],
                      "tflops": (work["flops_gu"] + work["flops_dn"]) / layer_s / 1e12},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s",
                    "h2d_bytes_per_step": T * d * 2 + T * E * 4,
                    "d2h_bytes_per_step": T * d * 4,
                    "how": "per layer one CUDA graph of the pinned H2D copies of x and scores, "
                           "the four calls and the D2H copy of out; synchronised every step"},
            "gpu_launches": 6 * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        del g_step, g_a, g_b, g_e2e
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
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="oracle seconds per step of the reference arm (default: fit ~1 min)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = synth.WORKLOADS[args.workload]
    if w.layers > 1:
        w = synth.Workload(w.name, w.T, w.E, w.k, w.d, w.f, w.routing, w.zipf_s, 1,
                           w.config_id, w.draw)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        synth.build()
        run_gpu(args, w)


if __name__ == "__main__":
    main()
