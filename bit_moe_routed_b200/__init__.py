"""bitmoe: routed-expert FFN of a DeepSeek-V4-Flash-style MoE layer on B200 (sm_100a).

Thin Python binding of the C ABI in ``include/bitmoe.h`` (libbitmoe.so).  It only
marshals arguments: torch provides device memory and the current CUDA stream, and
every step of the layer runs in the library's CUDA kernels.  There is no fallback:
if the library is missing or the device is not sm_100, calls raise.

    idx, w = route_topk(scores, k)              # step 1: top-k + sigmoid gate weights
    counts, offsets, perm, pos = dispatch(idx, E)  # step 2: stable grouping per expert
    y, y_sh = expert_ffn(x, k, weights, offsets, perm)  # steps 3-7 (FP4 x FP8 FFN)
    out = combine(y, y_sh, w, pos)              # step 8
    r = forward(x, scores, k, weights)          # all of it in one call (one kernel at T=1)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(_HERE, "libbitmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_WORKSPACE = -2
MOE_ERR_CUDA = -3
MOE_ERR_TIMEOUT = -4
MOE_ERR_UNSUPPORTED = -5
PATH_TILES, PATH_SINGLE, PATH_BATCHED, PATH_SINGLE_TC = 0, 1, 2, 3
MOE_NOALLOC_SCRATCH_BYTES = 24 << 20  # the fixed scratch of moe_expert_ffn_noalloc
GEMV_MAX_TOKENS = 64                  # default of moe_set_gemv_max_tokens

EXPORTS = (
    "moe_route_topk", "moe_dispatch", "moe_act_quant", "moe_expert_ffn", "moe_ffn_prepare",
    "moe_ffn_gate_up", "moe_ffn_down", "moe_combine", "moe_workspace_size", "moe_last_error",
    "moe_set_wait_limit_ns", "moe_sync_status", "moe_expert_ffn_noalloc",
    "moe_set_gemv_max_tokens", "moe_workspace_offsets", "moe_set_test_stall", "moe_forward",
    "moe_set_decode_engine", "moe_forward_path",
    "moe_ffn_path", "moe_router_topk", "moe_dispatch_workspace_size", "moe_forward_q2",
    "moe_fp8_gemm", "moe_fp8_gemm_workspace_size", "moe_shared_expert_fp8",
    "moe_shared_expert_fp8_workspace_size", "moe_shared_expert_fp8_offsets",
    "moe_expert_cache_reset", "moe_forward_streamed",
)


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"bitmoe error {code}: {msg}")
        self.code = code


class _Q2Experts(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales")]


class _Fp8Expert(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "gate", "gate_scales", "up", "up_scales", "down", "down_scales")] + [
        ("d", ctypes.c_int), ("f", ctypes.c_int)]


class _Weights(ctypes.Structure):
    _fields_ = [
        ("gate_codes", ctypes.c_void_p), ("gate_scales", ctypes.c_void_p),
        ("up_codes", ctypes.c_void_p), ("up_scales", ctypes.c_void_p),
        ("down_codes", ctypes.c_void_p), ("down_scales", ctypes.c_void_p),
        ("E", ctypes.c_int), ("d", ctypes.c_int), ("f", ctypes.c_int),
    ]


_lib = None


def lib():
    """Load libbitmoe.so (built in-tree by build.py); raise if it is not there."""
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(
                f"{SO} is missing: build it with `python -m bit_moe_routed_b200.build` "
                "(or __graft_entry__.build()); there is no fallback path")
        L = ctypes.CDLL(SO)
        P, I, Z, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
        W = ctypes.POINTER(_Weights)
        sig = {
            "moe_route_topk": [P, I, I, I, P, P, P],
            "moe_dispatch": [P, I, I, I, P, P, P, P, P, Z, P],
            "moe_act_quant": [P, I, I, P, P, P],
            "moe_expert_ffn": [P, I, I, W, P, P, P, P, P, Z, P],
            "moe_ffn_prepare": [P, I, I, W, P, P, P, Z, P],
            "moe_ffn_gate_up": [I, I, W, P, Z, P],
            "moe_ffn_down": [I, I, W, P, P, P, Z, P],
            "moe_combine": [P, P, P, P, I, I, I, P, P],
            "moe_workspace_size": [I, I, I, I, I],
            "moe_last_error": [],
            "moe_set_wait_limit_ns": [LL],
            "moe_sync_status": [P],
            "moe_expert_ffn_noalloc": [P, I, I, W, P, P, P, P, P],
            "moe_set_gemv_max_tokens": [I],
            "moe_set_decode_engine": [I],
            "moe_forward_path": [I, I, W],
            "moe_workspace_offsets": [I, I, I, I, I, P],
            "moe_set_test_stall": [I],
            "moe_forward": [P, P, I, I, W, P, P, P, P, P, P, P, P, P, P, Z, P],
            "moe_ffn_path": [I, I, W],
            "moe_router_topk": [P, P, I, I, I, I, P, P, P, P],
            "moe_dispatch_workspace_size": [I, I, I],
            "moe_forward_q2": [P, P, I, W, ctypes.POINTER(_Q2Experts), P, P, P, P, P, P, P, P,
                               P, P, Z, P],
            "moe_fp8_gemm": [P, P, I, I, P, P, I, P, P, Z, P],
            "moe_fp8_gemm_workspace_size": [I, I, I],
            "moe_shared_expert_fp8": [P, I, ctypes.POINTER(_Fp8Expert), P, P, Z, P],
            "moe_shared_expert_fp8_workspace_size": [I, I, I],
            "moe_shared_expert_fp8_offsets": [I, I, I, P],
            "moe_expert_cache_reset": [ctypes.POINTER(_ExpertCache), P],
            "moe_forward_streamed": [P, P, I, ctypes.POINTER(_HostExperts),
                                     ctypes.POINTER(_ExpertCache), P, P, P, P, P, P, P, P, P,
                                     P, Z, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.moe_workspace_size.restype = ctypes.c_size_t
        L.moe_dispatch_workspace_size.restype = ctypes.c_size_t
        L.moe_fp8_gemm_workspace_size.restype = ctypes.c_size_t
        L.moe_shared_expert_fp8_workspace_size.restype = ctypes.c_size_t
        L.moe_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(rc, lib().moe_last_error().decode(errors="replace"))


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _p(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to bitmoe must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


class _HostExperts(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales")]


class _ExpertCache(ctypes.Structure):
    _fields_ = [("slots", _Weights)] + [(n, ctypes.c_void_p) for n in (
        "slot_of", "expert_of", "last_use", "clock", "fetch", "stats")] + [("E", ctypes.c_int)]


@dataclass
class LayerWeights:
    """One layer's FP4 weights on the device, E+1 experts (index E = shared).

    gate_codes/up_codes [E+1, f, d/2] uint8, gate_scales/up_scales [E+1, f, d/32] uint8,
    down_codes [E+1, d, f/2] uint8, down_scales [E+1, d, f/32] uint8.
    """
    gate_codes: torch.Tensor
    gate_scales: torch.Tensor
    up_codes: torch.Tensor
    up_scales: torch.Tensor
    down_codes: torch.Tensor
    down_scales: torch.Tensor

    @property
    def E(self) -> int:
        return self.gate_codes.shape[0] - 1

    @property
    def f(self) -> int:
        return self.gate_codes.shape[1]

    @property
    def d(self) -> int:
        return self.gate_codes.shape[2] * 2

    def struct(self) -> _Weights:
        return _Weights(*(t.data_ptr() for t in (
            self.gate_codes, self.gate_scales, self.up_codes, self.up_scales, self.down_codes,
            self.down_scales)), self.E, self.d, self.f)

    @staticmethod
    def from_dict(d: dict) -> "LayerWeights":
        return LayerWeights(**{k: d[k] for k in (
            "gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales")})


@dataclass
class Q2Experts:
    """The E routed experts of a layer in the 2-bit codec on the device: gate_codes /
    up_codes [E, f, d/4], gate_scales / up_scales [E, f, d/128], down_codes [E, d, f/4],
    down_scales [E, d, f/128] (uint8)."""
    gate_codes: torch.Tensor
    gate_scales: torch.Tensor
    up_codes: torch.Tensor
    up_scales: torch.Tensor
    down_codes: torch.Tensor
    down_scales: torch.Tensor

    def struct(self) -> _Q2Experts:
        return _Q2Experts(*(t.data_ptr() for t in (
            self.gate_codes, self.gate_scales, self.up_codes, self.up_scales, self.down_codes,
            self.down_scales)))

    @staticmethod
    def from_dict(d: dict) -> "Q2Experts":
        return Q2Experts(**{k: d[k] for k in (
            "gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales")})


@dataclass
class Fp8Expert:
    """An FP8-weight expert on the device: gate / up [f, d] and down [d, f] e4m3 codes
    (uint8), gate_scales / up_scales [f/128, d/128] and down_scales [d/128, f/128] fp32."""
    gate: torch.Tensor
    gate_scales: torch.Tensor
    up: torch.Tensor
    up_scales: torch.Tensor
    down: torch.Tensor
    down_scales: torch.Tensor

    @property
    def d(self) -> int:
        return self.gate.shape[1]

    @property
    def f(self) -> int:
        return self.gate.shape[0]

    def struct(self) -> _Fp8Expert:
        return _Fp8Expert(*(t.data_ptr() for t in (
            self.gate, self.gate_scales, self.up, self.up_scales, self.down, self.down_scales)),
            self.d, self.f)

    @staticmethod
    def from_dict(d: dict) -> "Fp8Expert":
        return Fp8Expert(**{k: d[k] for k in (
            "gate", "gate_scales", "up", "up_scales", "down", "down_scales")})


def fp8_gemm(A: torch.Tensor, sa: torch.Tensor, B: torch.Tensor, sb: torch.Tensor,
             ws: torch.Tensor | None = None, stream=None, out: torch.Tensor | None = None):
    """C [M, N] fp32 = FP8 A [M, K] (scales sa [M, K/128]) times FP8 B [N, K] (scales
    sb [N/128, K/128]) transposed (moe_fp8_gemm)."""
    M, K = A.shape
    N = B.shape[0]
    if ws is None:
        n = int(lib().moe_fp8_gemm_workspace_size(M, N, K))
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=A.device)
    C = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=A.device)
    _check(lib().moe_fp8_gemm(_p(A), _p(sa), M, K, _p(B), _p(sb), N, _p(C), _p(ws), ws.numel(),
                              _stream(stream)))
    return C


def shared_expert_fp8(x: torch.Tensor, w: Fp8Expert, ws: torch.Tensor | None = None,
                      stream=None, out: torch.Tensor | None = None):
    """y_shared [T, d] fp32 of the FP8-weight expert for bf16 tokens x [T, d]
    (moe_shared_expert_fp8)."""
    T, d = x.shape
    if ws is None:
        n = int(lib().moe_shared_expert_fp8_workspace_size(T, w.d, w.f))
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=x.device)
    y = out if out is not None else torch.empty((T, d), dtype=torch.float32, device=x.device)
    st = w.struct()
    _check(lib().moe_shared_expert_fp8(_p(x), T, ctypes.byref(st), _p(y), _p(ws), ws.numel(),
                                       _stream(stream)))
    return y


def shared_expert_fp8_views(ws: torch.Tensor, T: int, d: int, f: int) -> dict:
    """Views of moe_shared_expert_fp8's intermediates in its workspace: qx, sx, h, qh, sh."""
    off = (ctypes.c_size_t * 5)()
    _check(lib().moe_shared_expert_fp8_offsets(T, d, f, off))
    u8 = lambda o, n: ws[o:o + n]  # noqa: E731
    f32 = lambda o, n: ws[o:o + 4 * n].view(torch.float32)  # noqa: E731
    return {"qx": u8(off[0], T * d).view(T, d), "sx": f32(off[1], T * (d // 128)).view(T, -1),
            "h": f32(off[2], T * f).view(T, f), "qh": u8(off[3], T * f).view(T, f),
            "sh": f32(off[4], T * (f // 128)).view(T, -1)}


_NAMES6 = ("gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales")


@dataclass
class HostExperts:
    """The E routed experts of a layer in pinned host memory (uint8 tensors with the
    LayerWeights layout, [E, ...] per matrix), which the device reads through unified
    addressing."""
    gate_codes: torch.Tensor
    gate_scales: torch.Tensor
    up_codes: torch.Tensor
    up_scales: torch.Tensor
    down_codes: torch.Tensor
    down_scales: torch.Tensor

    def struct(self) -> _HostExperts:
        return _HostExperts(*(getattr(self, n).data_ptr() for n in _NAMES6))

    @staticmethod
    def from_layer(w: "LayerWeights") -> "HostExperts":
        """Pinned host copies of a device layer's routed experts (expert E excluded)."""
        out = {}
        for n in _NAMES6:
            t = getattr(w, n)[:w.E]
            h = torch.empty(t.shape, dtype=torch.uint8, pin_memory=True)
            h.copy_(t)
            out[n] = h
        return HostExperts(**out)


class ExpertCache:
    """The HBM expert cache (moe_expert_cache_t): S + 1 slots (slot S holds the shared
    expert), the expert/slot tables, the LRU clock and the hit/miss counters."""

    def __init__(self, E: int, S: int, d: int, f: int, shared: "LayerWeights", device="cuda",
                 stream=None):
        self.E, self.S = E, S
        shp = {"gate_codes": (f, d // 2), "gate_scales": (f, d // 32), "up_codes": (f, d // 2),
               "up_scales": (f, d // 32), "down_codes": (d, f // 2), "down_scales": (d, f // 32)}
        sl = {}
        for n, (r, c) in shp.items():
            t = torch.empty((S + 1, r, c), dtype=torch.uint8, device=device)
            t[S].copy_(getattr(shared, n)[shared.E])  # the shared expert, resident
            sl[n] = t
        self.slots = LayerWeights(**sl)
        i32, i64 = torch.int32, torch.int64
        self.slot_of = torch.empty(E, dtype=i32, device=device)
        self.expert_of = torch.empty(S, dtype=i32, device=device)
        self.last_use = torch.empty(S, dtype=i64, device=device)
        self.clock = torch.empty(1, dtype=i64, device=device)
        self.fetch = torch.empty(1 + 2 * 32, dtype=i32, device=device)
        self.stats = torch.empty(2, dtype=i64, device=device)
        self.reset(stream)

    def struct(self) -> _ExpertCache:
        return _ExpertCache(self.slots.struct(), *(t.data_ptr() for t in (
            self.slot_of, self.expert_of, self.last_use, self.clock, self.fetch, self.stats)),
            self.E)

    def reset(self, stream=None) -> None:
        st = self.struct()
        _check(lib().moe_expert_cache_reset(ctypes.byref(st), _stream(stream)))


def forward_streamed(x: torch.Tensor, scores: torch.Tensor, k: int, host: HostExperts,
                     cache: ExpertCache, ws: torch.Tensor | None = None, stream=None,
                     outs: dict | None = None):
    """One token through the layer with the routed experts streamed from host memory
    through the cache (moe_forward_streamed); returns the dict of `forward`."""
    T, d = x.shape
    if T != 1:
        raise ValueError("moe_forward_streamed takes one token")
    E, f = cache.E, cache.slots.f
    dev = x.device
    if ws is None:
        ws = alloc_workspace(1, k, E, d, f, dev)
    o = dict(outs) if outs is not None else {}
    shapes = {"idx": ((1, k), torch.int32), "w": ((1, k), torch.float32),
              "counts": ((E,), torch.int32), "offsets": ((E + 1,), torch.int32),
              "perm": ((k,), torch.int32), "pos": ((k,), torch.int32),
              "y": ((k, d), torch.float32), "y_shared": ((1, d), torch.float32),
              "out": ((1, d), torch.float32)}
    for name, (shape, dtype) in shapes.items():
        if name not in o:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
    hs, cs = host.struct(), cache.struct()
    _check(lib().moe_forward_streamed(_p(scores), _p(x), k, ctypes.byref(hs), ctypes.byref(cs),
                                      _p(o["idx"]), _p(o["w"]), _p(o["counts"]),
                                      _p(o["offsets"]), _p(o["perm"]), _p(o["pos"]), _p(o["y"]),
                                      _p(o["y_shared"]), _p(o["out"]), _p(ws), ws.numel(),
                                      _stream(stream)))
    return dict(idx=o["idx"], w=o["w"], counts=o["counts"], offsets=o["offsets"],
                perm=o["perm"], pos=o["pos"], y=o["y"], y_shared=o["y_shared"], out=o["out"])


def set_wait_limit_ns(n: int) -> None:
    _check(lib().moe_set_wait_limit_ns(int(n)))


def set_test_stall(on: bool) -> None:
    """Testing knob: make the single-token FFN kernels' bounded wait run out (see the header)."""
    _check(lib().moe_set_test_stall(1 if on else 0))


def set_gemv_max_tokens(t: int) -> None:
    """Batches up to t tokens (at most 64) take the FP4 GEMV paths; 0 sends every batch to
    the tcgen05 tile kernels."""
    _check(lib().moe_set_gemv_max_tokens(int(t)))


def set_decode_engine(engine: int) -> None:
    """The single-token layer kernel of moe_forward: 0 (the default) on the CUDA cores, 1 on
    the tensor cores where the shapes allow it."""
    _check(lib().moe_set_decode_engine(int(engine)))


def sync_status(stream=None) -> None:
    _check(lib().moe_sync_status(_stream(stream)))


def workspace_size(T: int, k: int, E: int, d: int, f: int) -> int:
    return int(lib().moe_workspace_size(T, k, E, d, f))


def forward_path(T: int, k: int, w: "LayerWeights") -> int:
    """ffn_path for moe_forward: PATH_SINGLE_TC where the single-token layer kernel runs on
    the tensor cores."""
    st = w.struct()
    rc = lib().moe_forward_path(T, k, ctypes.byref(st))
    if rc < 0:
        _check(rc)
    return rc


def ffn_path(T: int, k: int, w: "LayerWeights") -> int:
    """PATH_TILES, PATH_SINGLE or PATH_BATCHED: the implementation moe_expert_ffn runs."""
    st = w.struct()
    rc = lib().moe_ffn_path(T, k, ctypes.byref(st))
    if rc < 0:
        _check(rc)
    return rc


def workspace_offsets(T: int, k: int, E: int, d: int, f: int) -> dict:
    """Byte offsets of qx, sx, qh, sh and h inside a workspace for (T, k, E, d, f); h is
    None when the layout keeps no fp32 hidden state."""
    off = (ctypes.c_size_t * 5)()
    _check(lib().moe_workspace_offsets(T, k, E, d, f, off))
    names = ("qx", "sx", "qh", "sh", "h")
    return {n: (None if v == ctypes.c_size_t(-1).value else int(v)) for n, v in zip(names, off)}


def workspace_views(ws: torch.Tensor, T: int, k: int, E: int, d: int, f: int) -> dict:
    """Views of the intermediate results moe_expert_ffn leaves in `ws` (rows: routed pairs
    in expert-sorted order, then the T shared-expert rows)."""
    o = workspace_offsets(T, k, E, d, f)
    R = T * k + T

    def view(name, n, dtype):
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return ws[o[name]:o[name] + nbytes].view(dtype)

    out = {"qx": view("qx", R * d, torch.uint8).view(R, d),
           "sx": view("sx", R * (d // 128), torch.float32).view(R, d // 128),
           "qh": view("qh", R * f, torch.uint8).view(R, f),
           "sh": view("sh", R * (f // 128), torch.float32).view(R, f // 128)}
    if o["h"] is not None:
        out["h"] = view("h", R * f, torch.float32).view(R, f)
    return out


def alloc_workspace(T: int, k: int, E: int, d: int, f: int, device="cuda") -> torch.Tensor:
    n = workspace_size(T, k, E, d, f)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def route_topk(scores: torch.Tensor, k: int, stream=None):
    T, E = scores.shape
    idx = torch.empty((T, k), dtype=torch.int32, device=scores.device)
    w = torch.empty((T, k), dtype=torch.float32, device=scores.device)
    _check(lib().moe_route_topk(_p(scores), T, E, k, _p(idx), _p(w), _stream(stream)))
    return idx, w


def router_topk(x: torch.Tensor, w_router: torch.Tensor, k: int, stream=None):
    """Router scores x . W_router^T (bf16 in, fp32 out) and their top-k: (scores, idx, w)."""
    T, d = x.shape
    E = w_router.shape[0]
    scores = torch.empty((T, E), dtype=torch.float32, device=x.device)
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(lib().moe_router_topk(_p(x), _p(w_router), T, d, E, k, _p(scores), _p(idx), _p(w),
                                 _stream(stream)))
    return scores, idx, w


def dispatch(idx: torch.Tensor, E: int, stream=None, multi: bool = True):
    """Stable grouping per expert; large batches use the multi-CTA form unless multi=False."""
    T, k = idx.shape
    dev = idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    pos = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    n = int(lib().moe_dispatch_workspace_size(T, k, E)) if multi else 0
    ws = torch.empty(max(n, 4), dtype=torch.uint8, device=dev) if n else None
    _check(lib().moe_dispatch(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(pos),
                              _p(ws), n, _stream(stream)))
    return counts, offsets, perm[:T * k], pos[:T * k]


def act_quant(x: torch.Tensor, stream=None):
    T, d = x.shape
    qx = torch.empty((T, d), dtype=torch.uint8, device=x.device)
    sx = torch.empty((T, d // 128), dtype=torch.float32, device=x.device)
    _check(lib().moe_act_quant(_p(x), T, d, _p(qx), _p(sx), _stream(stream)))
    return qx, sx


def expert_ffn(x: torch.Tensor, k: int, w: LayerWeights, offsets: torch.Tensor,
               perm: torch.Tensor, ws: torch.Tensor | None = None, out=None, stream=None):
    T, d = x.shape
    if ws is None:
        ws = alloc_workspace(T, k, w.E, w.d, w.f, x.device)
    if out is None:
        y = torch.empty((max(T * k, 1), d), dtype=torch.float32, device=x.device)
        ysh = torch.empty((max(T, 1), d), dtype=torch.float32, device=x.device)
    else:
        y, ysh = out
    ws_struct = w.struct()
    _check(lib().moe_expert_ffn(_p(x), T, k, ctypes.byref(ws_struct), _p(offsets), _p(perm),
                                _p(y), _p(ysh), _p(ws), ws.numel(), _stream(stream)))
    return y[:T * k], ysh[:T]


def expert_ffn_noalloc(x: torch.Tensor, k: int, w: LayerWeights, offsets: torch.Tensor,
                       perm: torch.Tensor, out=None, stream=None):
    """expert_ffn with the library's fixed device scratch instead of a workspace (for callers
    that cannot allocate; at most MOE_NOALLOC_SCRATCH_BYTES of scratch, calls must not
    overlap on the GPU)."""
    T, d = x.shape
    if out is None:
        y = torch.empty((max(T * k, 1), d), dtype=torch.float32, device=x.device)
        ysh = torch.empty((max(T, 1), d), dtype=torch.float32, device=x.device)
    else:
        y, ysh = out
    st = w.struct()
    _check(lib().moe_expert_ffn_noalloc(_p(x), T, k, ctypes.byref(st), _p(offsets), _p(perm),
                                        _p(y), _p(ysh), _stream(stream)))
    return y[:T * k], ysh[:T]


def ffn_prepare(x, k, w: LayerWeights, offsets, perm, ws, stream=None):
    T = x.shape[0]
    st = w.struct()
    _check(lib().moe_ffn_prepare(_p(x), T, k, ctypes.byref(st), _p(offsets), _p(perm), _p(ws),
                                 ws.numel(), _stream(stream)))


def ffn_gate_up(T, k, w: LayerWeights, ws, stream=None):
    st = w.struct()
    _check(lib().moe_ffn_gate_up(T, k, ctypes.byref(st), _p(ws), ws.numel(), _stream(stream)))


def ffn_down(T, k, w: LayerWeights, y, ysh, ws, stream=None):
    st = w.struct()
    _check(lib().moe_ffn_down(T, k, ctypes.byref(st), _p(y), _p(ysh), _p(ws), ws.numel(),
                              _stream(stream)))


def combine(y_routed: torch.Tensor, y_shared: torch.Tensor, w: torch.Tensor, pos: torch.Tensor,
            out: torch.Tensor | None = None, stream=None):
    T, k = w.shape
    d = y_shared.shape[1]
    if out is None:
        out = torch.empty((T, d), dtype=torch.float32, device=y_shared.device)
    _check(lib().moe_combine(_p(y_routed), _p(y_shared), _p(w), _p(pos), T, k, d, _p(out),
                             _stream(stream)))
    return out


def forward(x: torch.Tensor, scores: torch.Tensor, k: int, w: LayerWeights,
            ws: torch.Tensor | None = None, stream=None, outs: dict | None = None):
    """The whole layer in one call (moe_forward: one kernel for a single token, the four
    calls back to back otherwise); returns a dict of every output.  `outs` may hold
    preallocated outputs under the same names."""
    T, d = x.shape
    E = w.E
    dev = x.device
    if ws is None:
        ws = alloc_workspace(T, k, E, w.d, w.f, dev)
    o = dict(outs) if outs is not None else {}
    shapes = {"idx": ((T, k), torch.int32), "w": ((T, k), torch.float32),
              "counts": ((E,), torch.int32), "offsets": ((E + 1,), torch.int32),
              "perm": ((max(T * k, 1),), torch.int32), "pos": ((max(T * k, 1),), torch.int32),
              "y": ((max(T * k, 1), d), torch.float32), "y_shared": ((max(T, 1), d), torch.float32),
              "out": ((max(T, 1), d), torch.float32)}
    for name, (shape, dtype) in shapes.items():
        if name not in o:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
    st = w.struct()
    _check(lib().moe_forward(_p(scores), _p(x), T, k, ctypes.byref(st), _p(o["idx"]), _p(o["w"]),
                             _p(o["counts"]), _p(o["offsets"]), _p(o["perm"]), _p(o["pos"]),
                             _p(o["y"]), _p(o["y_shared"]), _p(o["out"]), _p(ws), ws.numel(),
                             _stream(stream)))
    return dict(idx=o["idx"], w=o["w"], counts=o["counts"], offsets=o["offsets"],
                perm=o["perm"][:T * k], pos=o["pos"][:T * k], y=o["y"][:T * k],
                y_shared=o["y_shared"][:T], out=o["out"][:T])


def forward_q2(x: torch.Tensor, scores: torch.Tensor, k: int, w: LayerWeights, q2: Q2Experts,
               ws: torch.Tensor | None = None, stream=None, outs: dict | None = None):
    """One token through the layer with 2-bit routed experts (moe_forward_q2): the routed
    experts from `q2`, the shared expert from `w` (FP4, index E).  Returns the dict of
    `forward`."""
    T, d = x.shape
    if T != 1:
        raise ValueError("moe_forward_q2 takes one token")
    E = w.E
    dev = x.device
    if ws is None:
        ws = alloc_workspace(1, k, E, w.d, w.f, dev)
    o = dict(outs) if outs is not None else {}
    shapes = {"idx": ((1, k), torch.int32), "w": ((1, k), torch.float32),
              "counts": ((E,), torch.int32), "offsets": ((E + 1,), torch.int32),
              "perm": ((k,), torch.int32), "pos": ((k,), torch.int32),
              "y": ((k, d), torch.float32), "y_shared": ((1, d), torch.float32),
              "out": ((1, d), torch.float32)}
    for name, (shape, dtype) in shapes.items():
        if name not in o:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
    st, qs = w.struct(), q2.struct()
    _check(lib().moe_forward_q2(_p(scores), _p(x), k, ctypes.byref(st), ctypes.byref(qs),
                                _p(o["idx"]), _p(o["w"]), _p(o["counts"]), _p(o["offsets"]),
                                _p(o["perm"]), _p(o["pos"]), _p(o["y"]), _p(o["y_shared"]),
                                _p(o["out"]), _p(ws), ws.numel(), _stream(stream)))
    return dict(idx=o["idx"], w=o["w"], counts=o["counts"], offsets=o["offsets"],
                perm=o["perm"], pos=o["pos"], y=o["y"], y_shared=o["y_shared"], out=o["out"])


def forward_calls(x: torch.Tensor, scores: torch.Tensor, k: int, w: LayerWeights,
                  ws: torch.Tensor | None = None, stream=None):
    """The whole layer through the four separate calls; returns a dict of every output."""
    idx, gw = route_topk(scores, k, stream)
    counts, offsets, perm, pos = dispatch(idx, w.E, stream)
    y, ysh = expert_ffn(x, k, w, offsets, perm, ws, stream=stream)
    out = combine(y, ysh, gw, pos, stream=stream)
    return dict(idx=idx, w=gw, counts=counts, offsets=offsets, perm=perm, pos=pos, y=y,
                y_shared=ysh, out=out)
