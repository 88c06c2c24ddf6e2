"""Oracle for the routed-expert MoE layer — TEST INFRASTRUCTURE ONLY.

Python front end (ctypes + numpy) for the plain C oracle in ``oracle.c``.  Only
the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline /
reference legs may import this package; the product library never does.  It
shares no code with the CUDA library.  See ``oracle.h`` for the passages each
function follows.

Parity pins live in ``tests/test_oracle_*.py``: format tables against the OCP MX
v1.0 values and torch's float8 decoders, the e4m3 encoder against brute force,
routing and dispatch against torch.topk / stable torch.sort, the FP4 GEMV on
integer-exact inputs against int64 numpy, the FFN at k = 1 against a dense
float64 FFN assembled from library routines, and token-permutation invariance.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(_HERE, "liboracle.so")
_SRC = [os.path.join(_HERE, "oracle.c"), os.path.join(_HERE, "oracle.h")]


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (plain C99 + OpenMP, no fp contraction)."""
    newest = max(os.path.getmtime(p) for p in _SRC)
    if force or not os.path.exists(SO) or os.path.getmtime(SO) < newest:
        subprocess.check_call([
            "gcc", "-O2", "-std=c99", "-D_DEFAULT_SOURCE", "-fPIC", "-shared", "-fopenmp",
            "-ffp-contract=off", "-fno-fast-math", "-o", SO, _SRC[0], "-lm"])
    return SO


FP4, Q2, FP8 = 0, 1, 2  # weight codecs (oracle.h: ORACLE_FP4, ORACLE_Q2, ORACLE_FP8)


class _Expert(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales")] + [
        ("codec", ctypes.c_int)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(SO)
        P = ctypes.c_void_p
        I = ctypes.c_int
        L.oracle_e2m1_value.argtypes = [I]
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [I]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_ue8m0_value.argtypes = [I]
        L.oracle_ue8m0_value.restype = ctypes.c_double
        L.oracle_q2_value.argtypes = [I]
        L.oracle_q2_value.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_quant_blocks.argtypes = [P, I, P, P]
        L.oracle_act_quant.argtypes = [P, I, I, P, P]
        L.oracle_route_topk.argtypes = [P, I, I, I, P, P]
        L.oracle_router_scores.argtypes = [P, P, I, I, I, P]
        L.oracle_dispatch.argtypes = [P, I, I, I, P, P, P, P]
        L.oracle_fp4_gemv.argtypes = [P, P, I, I, P, P]
        L.oracle_q2_gemv.argtypes = [P, P, I, I, P, P]
        L.oracle_fp8_gemm.argtypes = [P, P, I, P, P, I, I, P]
        L.oracle_expert_ffn.argtypes = [ctypes.POINTER(_Expert), I, I, P, P, I, P, P, P]
        L.oracle_expert_ffn_h.argtypes = [ctypes.POINTER(_Expert), I, I, P, P, I, P, P, P, P]
        L.oracle_combine_token.argtypes = [P, P, P, I, I, P]
        L.oracle_moe_tokens.argtypes = [P, I, I, I, I, I, ctypes.POINTER(_Expert), P, P, P, I,
                                        P, P, P]
        L.oracle_moe_layer.argtypes = [P, I, I, I, I, I, ctypes.POINTER(_Expert), P, P, P, P, P]
        L.oracle_set_threads.argtypes = [I]
        L.oracle_get_threads.restype = I
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# ---- formats ----------------------------------------------------------------------
def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def ue8m0_value(code: int) -> float:
    return lib().oracle_ue8m0_value(int(code))


def q2_value(code: int) -> float:
    return lib().oracle_q2_value(int(code))


def e4m3_encode(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float32).ravel()
    return np.array([lib().oracle_e4m3_encode(float(x)) for x in v], dtype=np.uint8)


def quant_blocks(v: np.ndarray):
    v, pv = _c(v, np.float32)
    n = v.size
    q = np.empty(n, np.uint8)
    s = np.empty(n // 128, np.float32)
    lib().oracle_quant_blocks(pv, n, q.ctypes.data, s.ctypes.data)
    return q, s


# ---- layer steps --------------------------------------------------------------------
def _bf16_bits(x) -> np.ndarray:
    """bf16 torch tensor or uint16 numpy array -> uint16 numpy array of the bit patterns."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        return x.contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(x, dtype=np.uint16)


def act_quant(x):
    xb = _bf16_bits(x)
    T, d = xb.shape
    q = np.empty((T, d), np.uint8)
    s = np.empty((T, d // 128), np.float32)
    lib().oracle_act_quant(xb.ctypes.data, T, d, q.ctypes.data, s.ctypes.data)
    return q, s


def router_scores(x, w_router) -> np.ndarray:
    """scores [T, E] (double) = x [T, d] . W_router [E, d]^T over bf16 inputs."""
    xb = _bf16_bits(x)
    wb = _bf16_bits(w_router)
    T, d = xb.shape
    E = wb.shape[0]
    out = np.empty((T, E), np.float64)
    lib().oracle_router_scores(xb.ctypes.data, wb.ctypes.data, T, d, E, out.ctypes.data)
    return out


def route_topk(scores: np.ndarray, k: int):
    s, ps = _c(scores, np.float32)
    T, E = s.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lib().oracle_route_topk(ps, T, E, k, idx.ctypes.data, w.ctypes.data)
    return idx, w


def dispatch(idx: np.ndarray, E: int):
    idx, pi = _c(idx, np.int32)
    T, k = idx.shape
    P = T * k
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(max(P, 1), np.int32)
    pos = np.empty(max(P, 1), np.int32)
    lib().oracle_dispatch(pi, T, k, E, counts.ctypes.data, offsets.ctypes.data,
                          perm.ctypes.data, pos.ctypes.data)
    return counts, offsets, perm[:P], pos[:P]


def fp4_gemv(codes: np.ndarray, scales: np.ndarray, xhat: np.ndarray) -> np.ndarray:
    codes, pc = _c(codes, np.uint8)
    scales, psc = _c(scales, np.uint8)
    xhat, px = _c(xhat, np.float64)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty(rows, np.float64)
    lib().oracle_fp4_gemv(pc, psc, rows, K, px, out.ctypes.data)
    return out


def q2_gemv(codes: np.ndarray, scales: np.ndarray, xhat: np.ndarray) -> np.ndarray:
    """2-bit matrix (codes [rows, K/4], scales [rows, K/128]) times xhat, in double."""
    codes, pc = _c(codes, np.uint8)
    scales, psc = _c(scales, np.uint8)
    xhat, px = _c(xhat, np.float64)
    rows, K = codes.shape[0], codes.shape[1] * 4
    out = np.empty(rows, np.float64)
    lib().oracle_q2_gemv(pc, psc, rows, K, px, out.ctypes.data)
    return out


def fp8_gemm(A: np.ndarray, sa: np.ndarray, B: np.ndarray, sb: np.ndarray) -> np.ndarray:
    """C [M, N] (double) = (e4m3(A) * sa per 128-block) . (e4m3(B) * sb per 128x128 block)^T;
    A [M, K], B [N, K] e4m3 codes, sa [M, K/128], sb [N/128, K/128] fp32."""
    A, pa = _c(A, np.uint8)
    B, pb = _c(B, np.uint8)
    sa, psa = _c(sa, np.float32)
    sb, psb = _c(sb, np.float32)
    M, K = A.shape
    N = B.shape[0]
    C = np.empty((M, N), np.float64)
    lib().oracle_fp8_gemm(pa, psa, M, pb, psb, N, K, C.ctypes.data)
    return C


class ExpertSet:
    """Holds numpy weight arrays alive and exposes a ctypes array of experts.

    ``experts`` maps expert index -> object with gate_codes, gate_scales, up_codes,
    up_scales, down_codes, down_scales (uint8 numpy arrays) and optionally ``codec``
    (FP4 when absent); missing experts are NULL.
    """

    def __init__(self, n: int, experts: dict):
        self._keep = []
        self.arr = (_Expert * n)()
        for e, ex in experts.items():
            vals = []
            codec = int(getattr(ex, "codec", FP4))
            for name in ("gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes",
                         "down_scales"):
                dt = np.float32 if (codec == FP8 and name.endswith("scales")) else np.uint8
                a = np.ascontiguousarray(getattr(ex, name), dtype=dt)
                self._keep.append(a)
                vals.append(a.ctypes.data)
            self.arr[e] = _Expert(*vals, int(getattr(ex, "codec", FP4)))


def expert_ffn(ex, d: int, f: int, qx: np.ndarray, sx: np.ndarray, want_h: bool = False):
    es = ExpertSet(1, {0: ex})
    qx, pq = _c(qx, np.uint8)
    sx, ps = _c(sx, np.float32)
    ntok = qx.shape[0]
    y = np.empty((ntok, d), np.float64)
    hq = np.empty((ntok, f), np.uint8) if want_h else None
    hs = np.empty((ntok, f // 128), np.float32) if want_h else None
    lib().oracle_expert_ffn(es.arr, d, f, pq, ps, ntok, y.ctypes.data,
                            hq.ctypes.data if want_h else None,
                            hs.ctypes.data if want_h else None)
    return (y, hq, hs) if want_h else y


def expert_ffn_h(ex, d: int, f: int, qx: np.ndarray, sx: np.ndarray):
    """(y [ntok, d], h codes [ntok, f], h scales [ntok, f/128], h fp32 before quantisation)."""
    es = ExpertSet(1, {0: ex})
    qx, pq = _c(qx, np.uint8)
    sx, ps = _c(sx, np.float32)
    ntok = qx.shape[0]
    y = np.empty((ntok, d), np.float64)
    hq = np.empty((ntok, f), np.uint8)
    hs = np.empty((ntok, f // 128), np.float32)
    hf = np.empty((ntok, f), np.float32)
    lib().oracle_expert_ffn_h(es.arr, d, f, pq, ps, ntok, y.ctypes.data, hq.ctypes.data,
                              hs.ctypes.data, hf.ctypes.data)
    return y, hq, hs, hf


def combine(y_sh: np.ndarray, y_pair: np.ndarray, w: np.ndarray) -> np.ndarray:
    """out[t] = y_sh[t] + sum_j w[t,j] y_pair[t,j]; y_pair [T, k, d]."""
    T, k, d = y_pair.shape
    out = np.empty((T, d), np.float64)
    ysh, _ = _c(y_sh, np.float64)
    yp, _ = _c(y_pair, np.float64)
    ww, _ = _c(w, np.float64)
    for t in range(T):
        lib().oracle_combine_token(ysh[t].ctypes.data, yp[t].ctypes.data, ww[t].ctypes.data, k,
                                   d, out[t].ctypes.data)
    return out


def moe_tokens(x, E: int, k: int, d: int, f: int, experts: dict, idx: np.ndarray,
               w: np.ndarray, tokens):
    """Layer output for selected tokens: (y_pair [n,k,d], y_sh [n,d], out [n,d])."""
    xb = _bf16_bits(x)
    T = xb.shape[0]
    es = ExpertSet(E + 1, experts)
    idx, pi = _c(idx, np.int32)
    w, pw = _c(w, np.float64)
    tok, pt = _c(np.asarray(tokens), np.int32)
    n = tok.size
    y_pair = np.empty((n, k, d), np.float64)
    y_sh = np.empty((n, d), np.float64)
    out = np.empty((n, d), np.float64)
    lib().oracle_moe_tokens(xb.ctypes.data, T, d, f, E, k, es.arr, pi, pw, pt, n,
                            y_pair.ctypes.data, y_sh.ctypes.data, out.ctypes.data)
    return y_pair, y_sh, out


def moe_layer(x, E: int, k: int, d: int, f: int, experts: dict, idx: np.ndarray,
              w: np.ndarray):
    """Whole layer: (y_pair [T*k, d] in pair order, y_sh [T, d], out [T, d])."""
    xb = _bf16_bits(x)
    T = xb.shape[0]
    es = ExpertSet(E + 1, experts)
    idx, pi = _c(idx, np.int32)
    w, pw = _c(w, np.float64)
    y_pair = np.empty((T * k, d), np.float64)
    y_sh = np.empty((T, d), np.float64)
    out = np.empty((T, d), np.float64)
    lib().oracle_moe_layer(xb.ctypes.data, T, d, f, E, k, es.arr, pi, pw, y_pair.ctypes.data,
                           y_sh.ctypes.data, out.ctypes.data)
    return y_pair, y_sh, out


# ---- expert cache (NEXT-4: routed experts streamed from host memory) -----------------
def lru_cache_steps(selections, E: int, S: int):
    """The expert cache's decisions over a sequence of steps, plainly: a cache of S slots,
    each holding one routed expert or nothing; at step n (n = 1, 2, ...) the selected
    experts, taken in ascending id, are first marked used (hits), then each expert not
    resident gets the least recently used slot (smallest last-use step, ties to the lower
    slot; empty slots count as never used) among the slots not holding an expert of this
    step, whose expert is evicted.  (dpshk.com article, "核心实现一": experts are read as
    they are needed and kept under an LRU share.)  Returns, per step, (hits, misses, fills)
    with fills = [(expert, slot)], and the final (slot_of [E], expert_of [S], last_use [S]).
    """
    slot_of = [-1] * E
    expert_of = [-1] * S
    last_use = [0] * S
    out = []
    for n, sel in enumerate(selections, start=1):
        sel = sorted(set(int(e) for e in sel))
        hits, misses, fills = [], [], []
        for e in sel:
            if slot_of[e] >= 0:
                last_use[slot_of[e]] = n
                hits.append(e)
        for e in sel:
            if slot_of[e] >= 0:
                continue
            best = None
            for s in range(S):
                if expert_of[s] in sel:
                    continue
                if best is None or last_use[s] < last_use[best]:
                    best = s
            if best is None:
                raise ValueError("fewer slots than selected experts")
            if expert_of[best] >= 0:
                slot_of[expert_of[best]] = -1
            expert_of[best] = e
            slot_of[e] = best
            last_use[best] = n
            misses.append(e)
            fills.append((e, best))
        out.append((hits, misses, fills))
    return out, (slot_of, expert_of, last_use)
