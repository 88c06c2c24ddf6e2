"""Seeded synthetic inputs for the routed-expert MoE layer.

This module generates inputs only and holds none of the method's arithmetic:
  * FP4 code bytes and UE8M0 scale bytes of the expert weights
    (SplitMix64, see synth_host.c / synth_dev.cu),
  * token activations x ~ N(0, 1) rounded to bf16,
  * router scores, either uniform (U[0,1) + e * 1e-6) or Zipf(s)-popular
    experts through Gumbel noise (Kool, van Hoof, Welling, "Stochastic Beams
    and Where to Find Them", ICML 2019: the top-k of log p + Gumbel(0,1) is a
    sample of k experts without replacement from p).

Both the oracle side (tests, CPU baseline) and the CUDA side (tests, bench)
draw their inputs here.  Weights are a pure function of (seed, layer, expert,
matrix, byte index).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(_HERE, "libsynth_host.so")
DEV_SO = os.path.join(_HERE, "libsynth_dev.so")

GATE, UP, DOWN = 0, 1, 2
CODES, SCALES = 0, 1


# --------------------------------------------------------------------------------------
# Workloads (the layer shapes the pages' model uses: 256 routed experts + 1 shared,
# top-6, 43 layers; hidden 4096, expert width 2048).
# --------------------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    E: int
    k: int
    d: int
    f: int
    routing: str = "uniform"  # "uniform" or "zipf"
    zipf_s: float = 1.0
    layers: int = 1
    config_id: int = 0
    draw: int = 0
    routed_codec: str = "fp4"  # "fp4", or "q2": routed experts in the 2-bit codec

    def seed(self, layer: int = 0) -> int:
        return 1000 * self.config_id + 10 * self.draw + layer


WORKLOADS = {
    "tiny": Workload("tiny", T=4, E=8, k=2, d=256, f=128, config_id=0),
    "decode_t1": Workload("decode_t1", T=1, E=256, k=6, d=4096, f=2048, config_id=1),
    "decode_t64_zipf": Workload("decode_t64_zipf", T=64, E=256, k=6, d=4096, f=2048,
                                routing="zipf", zipf_s=1.0, config_id=2),
    "prefill_t4096_uniform": Workload("prefill_t4096_uniform", T=4096, E=256, k=6, d=4096,
                                      f=2048, config_id=3, draw=0),
    "prefill_t4096_zipf": Workload("prefill_t4096_zipf", T=4096, E=256, k=6, d=4096, f=2048,
                                   routing="zipf", zipf_s=1.2, config_id=3, draw=1),
    # decode_t1's token, scores and shared expert with the routed experts in the 2-bit
    # codec (the deployed model of the ai-muninn.com post: IQ2_XXS routed experts)
    "decode_t1_q2": Workload("decode_t1_q2", T=1, E=256, k=6, d=4096, f=2048, config_id=1,
                             routed_codec="q2"),
    "layers43_t1": Workload("layers43_t1", T=1, E=256, k=6, d=4096, f=2048, routing="zipf",
                            zipf_s=1.0, layers=43, config_id=4, draw=0),
    "layers43_t32": Workload("layers43_t32", T=32, E=256, k=6, d=4096, f=2048,
                             routing="zipf", zipf_s=1.0, layers=43, config_id=4, draw=1),
}


def matrix_shape(which: int, d: int, f: int):
    """(rows, reduction length) of one expert matrix: gate/up are [f, d], down is [d, f]."""
    return (f, d) if which in (GATE, UP) else (d, f)


def code_bytes(which: int, d: int, f: int) -> int:
    r, K = matrix_shape(which, d, f)
    return r * K // 2


def scale_bytes(which: int, d: int, f: int) -> int:
    r, K = matrix_shape(which, d, f)
    return r * K // 32


def expert_bytes(d: int, f: int) -> int:
    return sum(code_bytes(m, d, f) + scale_bytes(m, d, f) for m in (GATE, UP, DOWN))


# --------------------------------------------------------------------------------------
# Native builds (plain gcc for the host generator, nvcc for the device fill).
# --------------------------------------------------------------------------------------
def build(device: bool = True) -> None:
    src = os.path.join(_HERE, "synth_host.c")
    if not os.path.exists(HOST_SO) or os.path.getmtime(HOST_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", HOST_SO, src])
    if device:
        dsrc = os.path.join(_HERE, "synth_dev.cu")
        if not os.path.exists(DEV_SO) or os.path.getmtime(DEV_SO) < os.path.getmtime(dsrc):
            subprocess.check_call([
                "nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                "-Xcompiler", "-fPIC", "-shared", "-o", DEV_SO, dsrc])


_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        build(device=False)
        lib = ctypes.CDLL(HOST_SO)
        lib.synth_fill.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_size_t]
        lib.synth_fill.restype = None
        lib.synth_word.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_word.restype = ctypes.c_uint64
        lib.synth_stream_id.argtypes = [ctypes.c_int] * 4
        lib.synth_stream_id.restype = ctypes.c_uint64
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(DEV_SO):
            raise RuntimeError(f"device weight generator not built: {DEV_SO} (run build())")
        lib = ctypes.CDLL(DEV_SO)
        lib.synth_fill_dev.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p,
                                       ctypes.c_void_p]
        lib.synth_fill_dev.restype = ctypes.c_int
        _dev = lib
    return _dev


# --------------------------------------------------------------------------------------
# Weights
# --------------------------------------------------------------------------------------
def expert_matrix_host(seed: int, layer: int, expert: int, which: int, kind: int, d: int,
                       f: int) -> np.ndarray:
    """One expert matrix as a uint8 array: codes [rows, K/2] or scales [rows, K/32]."""
    r, K = matrix_shape(which, d, f)
    cols = K // 2 if kind == CODES else K // 32
    out = np.empty((r, cols), dtype=np.uint8)
    _host_lib().synth_fill(seed, layer, expert, which, kind, out.ctypes.data, 0, out.size)
    return out


@dataclass
class HostExpert:
    """Codes and scales of one expert's three matrices (numpy uint8)."""
    gate_codes: np.ndarray
    gate_scales: np.ndarray
    up_codes: np.ndarray
    up_scales: np.ndarray
    down_codes: np.ndarray
    down_scales: np.ndarray


def host_expert(seed: int, layer: int, expert: int, d: int, f: int) -> HostExpert:
    g = lambda m, k: expert_matrix_host(seed, layer, expert, m, k, d, f)  # noqa: E731
    return HostExpert(g(GATE, CODES), g(GATE, SCALES), g(UP, CODES), g(UP, SCALES),
                      g(DOWN, CODES), g(DOWN, SCALES))


def host_layer_weights(seed: int, layer: int, E: int, d: int, f: int):
    """All E+1 experts of a layer stacked per matrix: dict name -> uint8 [E+1, rows, cols]."""
    out = {}
    for name, which in (("gate", GATE), ("up", UP), ("down", DOWN)):
        for kind, suffix in ((CODES, "codes"), (SCALES, "scales")):
            out[f"{name}_{suffix}"] = np.stack([
                expert_matrix_host(seed, layer, e, which, kind, d, f) for e in range(E + 1)])
    return out


def device_layer_weights(seed: int, layer: int, E: int, d: int, f: int, device="cuda",
                         stream=None):
    """All E+1 experts of a layer generated in device memory (torch uint8 tensors)."""
    lib = _dev_lib()
    out = {}
    s = stream if stream is not None else torch.cuda.current_stream(device)
    for name, which in (("gate", GATE), ("up", UP), ("down", DOWN)):
        r, K = matrix_shape(which, d, f)
        for kind, suffix, cols in ((CODES, "codes", K // 2), (SCALES, "scales", K // 32)):
            t = torch.empty((E + 1, r, cols), dtype=torch.uint8, device=device)
            rc = lib.synth_fill_dev(seed, layer, E + 1, which, kind, r * cols, t.data_ptr(),
                                    ctypes.c_void_p(s.cuda_stream))
            if rc != 0:
                raise RuntimeError(f"synth_fill_dev failed: {rc}")
            out[f"{name}_{suffix}"] = t
    return out


# --------------------------------------------------------------------------------------
# 2-bit routed-expert weights: codes [rows, K/4] (four 2-bit codes per byte) and scales
# [rows, K/128], drawn by the same generator as the FP4 bytes from seeds seed ^ Q2_SEED
# (other streams than the FP4 weights of the same layer).  Any byte is four valid codes;
# scale bytes are 121 + (byte AND 3), as for FP4.
# --------------------------------------------------------------------------------------
Q2_SEED = 0x5132


def q2_cols(which: int, kind: int, d: int, f: int) -> int:
    r, K = matrix_shape(which, d, f)
    return K // 4 if kind == CODES else K // 128


def expert_matrix_host_q2(seed: int, layer: int, expert: int, which: int, kind: int, d: int,
                          f: int) -> np.ndarray:
    r, _ = matrix_shape(which, d, f)
    out = np.empty((r, q2_cols(which, kind, d, f)), dtype=np.uint8)
    _host_lib().synth_fill(seed ^ Q2_SEED, layer, expert, which, kind, out.ctypes.data, 0,
                           out.size)
    return out


def host_expert_q2(seed: int, layer: int, expert: int, d: int, f: int) -> HostExpert:
    g = lambda m, k: expert_matrix_host_q2(seed, layer, expert, m, k, d, f)  # noqa: E731
    return HostExpert(g(GATE, CODES), g(GATE, SCALES), g(UP, CODES), g(UP, SCALES),
                      g(DOWN, CODES), g(DOWN, SCALES))


def device_layer_weights_q2(seed: int, layer: int, E: int, d: int, f: int, device="cuda",
                            stream=None):
    """The E routed experts of a layer in the 2-bit codec, in device memory (torch uint8
    tensors [E, rows, cols]); the same bytes as host_expert_q2."""
    lib = _dev_lib()
    out = {}
    s = stream if stream is not None else torch.cuda.current_stream(device)
    for name, which in (("gate", GATE), ("up", UP), ("down", DOWN)):
        r, _ = matrix_shape(which, d, f)
        for kind, suffix in ((CODES, "codes"), (SCALES, "scales")):
            cols = q2_cols(which, kind, d, f)
            t = torch.empty((E, r, cols), dtype=torch.uint8, device=device)
            rc = lib.synth_fill_dev(seed ^ Q2_SEED, layer, E, which, kind, r * cols, t.data_ptr(),
                                    ctypes.c_void_p(s.cuda_stream))
            if rc != 0:
                raise RuntimeError(f"synth_fill_dev failed: {rc}")
            out[f"{name}_{suffix}"] = t
    return out


# --------------------------------------------------------------------------------------
# FP8 shared expert: e4m3 codes [rows, K] and fp32 scales [rows/128, K/128], from the same
# generator with seeds seed ^ FP8_SEED.  A code byte b becomes (b AND 0x87) OR
# ((4 + ((b >> 3) AND 7)) << 3): sign and mantissa from b, exponent field 4..11 (values
# 2^-3 .. 15, no NaN); a scale is 2^(e - 127) with e the generator's scale byte (121..124).
# --------------------------------------------------------------------------------------
FP8_SEED = 0xF8F8


def _fp8_codes(raw):
    return (raw & 0x87) | ((4 + ((raw >> 3) & 7)) << 3)


def host_expert_fp8(seed: int, layer: int, d: int, f: int) -> dict:
    """The FP8 shared expert as numpy arrays: gate/up/down codes (uint8) and scales
    (float32); drawn from the streams of expert 0 under the FP8 seed."""
    out = {}
    for name, which in (("gate", GATE), ("up", UP), ("down", DOWN)):
        r, K = matrix_shape(which, d, f)
        raw = np.empty((r, K), np.uint8)
        _host_lib().synth_fill(seed ^ FP8_SEED, layer, 0, which, CODES, raw.ctypes.data, 0,
                               raw.size)
        sb = np.empty((r // 128, K // 128), np.uint8)
        _host_lib().synth_fill(seed ^ FP8_SEED, layer, 0, which, SCALES, sb.ctypes.data, 0,
                               sb.size)
        out[name] = _fp8_codes(raw).astype(np.uint8)
        out[f"{name}_scales"] = np.ldexp(1.0, sb.astype(np.int32) - 127).astype(np.float32)
    return out


def device_expert_fp8(seed: int, layer: int, d: int, f: int, device="cuda",
                      stream=None) -> dict:
    """The same expert generated in device memory (torch tensors)."""
    lib = _dev_lib()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    out = {}
    for name, which in (("gate", GATE), ("up", UP), ("down", DOWN)):
        r, K = matrix_shape(which, d, f)
        raw = torch.empty((r, K), dtype=torch.uint8, device=device)
        sb = torch.empty((r // 128, K // 128), dtype=torch.uint8, device=device)
        for t, kind in ((raw, CODES), (sb, SCALES)):
            rc = lib.synth_fill_dev(seed ^ FP8_SEED, layer, 1, which, kind, t.numel(),
                                    t.data_ptr(), ctypes.c_void_p(s.cuda_stream))
            if rc != 0:
                raise RuntimeError(f"synth_fill_dev failed: {rc}")
        with torch.cuda.stream(s):
            out[name] = _fp8_codes(raw.to(torch.int32)).to(torch.uint8)
            out[f"{name}_scales"] = torch.ldexp(torch.ones_like(sb, dtype=torch.float32),
                                                sb.to(torch.int32) - 127)
    return out


def fp8_expert_bytes(d: int, f: int) -> int:
    return 3 * d * f + 3 * (d // 128) * (f // 128) * 4


def q2_expert_bytes(d: int, f: int) -> int:
    return sum(matrix_shape(m, d, f)[0] * (q2_cols(m, CODES, d, f) + q2_cols(m, SCALES, d, f))
               for m in (GATE, UP, DOWN))


# --------------------------------------------------------------------------------------
# Activations and router scores (torch CPU generators, fp32 then rounded where stated)
# --------------------------------------------------------------------------------------
def gen_x(T: int, d: int, seed: int) -> torch.Tensor:
    """x ~ N(0,1) drawn in fp32, rounded to bf16; shape [T, d]."""
    g = torch.Generator().manual_seed(int(seed) * 2 + 1)
    return torch.randn(T, d, generator=g, dtype=torch.float32).to(torch.bfloat16)


def _make_distinct(s: torch.Tensor) -> torch.Tensor:
    """Break exact fp32 ties inside each row: among equal values, every one but the
    lowest expert index is moved down by one ulp (repeated until the row is distinct).
    Ties are rare (birthday collisions of fp32 draws); the change is one ulp."""
    s = s.clone()
    for _ in range(64):
        vals, order = torch.sort(s, dim=1, stable=True)
        dup = torch.zeros_like(vals, dtype=torch.bool)
        dup[:, 1:] = vals[:, 1:] == vals[:, :-1]
        if not bool(dup.any()):
            return s
        rows, cols = torch.nonzero(dup, as_tuple=True)
        e = order[rows, cols]
        s[rows, e] = torch.nextafter(s[rows, e], torch.tensor(-float("inf")))
    raise RuntimeError("could not make scores distinct")


def gen_scores_uniform(T: int, E: int, seed: int) -> torch.Tensor:
    """scores[t, e] = U[0,1) + e * 1e-6 (fp32), ties broken by one ulp."""
    g = torch.Generator().manual_seed(int(seed) * 2 + 2)
    s = torch.rand(T, E, generator=g, dtype=torch.float32) + \
        torch.arange(E, dtype=torch.float32) * 1e-6
    return _make_distinct(s)


def gen_scores_zipf(T: int, E: int, s_exp: float, seed: int) -> torch.Tensor:
    """scores[t, e] = log p_e + Gumbel(0,1), p_{pi(r)} ~ r^-s over a seeded expert permutation."""
    g = torch.Generator().manual_seed(int(seed) * 2 + 2)
    perm = torch.randperm(E, generator=g)
    rank = torch.empty(E, dtype=torch.float64)
    rank[perm] = torch.arange(1, E + 1, dtype=torch.float64)
    logp = -s_exp * torch.log(rank)
    logp = logp - torch.logsumexp(logp, 0)
    u = torch.rand(T, E, generator=g, dtype=torch.float64).clamp_min(1e-300)
    gumbel = -torch.log(-torch.log(u))
    return _make_distinct((logp[None, :] + gumbel).to(torch.float32))


def gen_scores(w: Workload, layer: int = 0) -> torch.Tensor:
    if w.routing == "zipf":
        return gen_scores_zipf(w.T, w.E, w.zipf_s, w.seed(layer))
    return gen_scores_uniform(w.T, w.E, w.seed(layer))


def gen_router_weights(E: int, d: int, seed: int) -> torch.Tensor:
    """W_router [E, d]: N(0, 1/d) drawn in fp32, rounded to bf16 (scores of unit-variance
    tokens then have unit variance)."""
    g = torch.Generator().manual_seed(int(seed) * 2 + 3)
    return (torch.randn(E, d, generator=g, dtype=torch.float32) / math.sqrt(d)).to(torch.bfloat16)


def gen_layer_inputs(w: Workload, layer: int = 0):
    """(x bf16 [T, d], scores fp32 [T, E]) for one layer of a workload, on the CPU."""
    return gen_x(w.T, w.d, w.seed(layer)), gen_scores(w, layer)
