"""Shared helpers for the parity tests: seeded inputs for both sides, oracle references,
and the comparison rules.

Integers and codes (routing indices, dispatch permutation, activation codes and scales)
must match bit-exactly.  Floating-point outputs are compared in two steps, because the
method re-quantises the hidden state h = silu(g) * u to e4m3 (3 mantissa bits) from fp32
and an element of h that lies next to an e4m3 rounding midpoint may round either way on
a correct implementation:

1. h codes.  The GPU's re-quantised h (codes qh and scales sh, read from the workspace)
   must equal the oracle's, except for elements where the two differ by one code step
   AND the oracle's value h/s lies within a derived error window of the midpoint between
   the two codes.  The window comes from an a-priori bound on the GPU's fp32 error, not
   from observed GPU behaviour (``h_error_bound``):
     - g and u are fp32 dot products over K = d; every product of an e2m1 value, a power
       of two and an e4m3 value is exact in fp32, so the error is that of the sums.  A
       product passes through at most D = 128 + K/128 + 8 roundings on its way to the
       result (<= 128 inside a 128-element chunk, whatever order the tensor core or the
       MMA chain adds in; one fused multiply-add per chunk when the chunk is scaled by
       the activation's fp32 block scale and added to the total; <= 8 to combine K-split
       partials).  Each rounding errs by at most 2^-23 of its result (truncation
       included), so |dg| <= D * 2^-23 * sum_k |W[n,k] x[k]| and likewise for u
       (standard forward error bound of summation, gamma_D).
     - h = g / (1 + exp(-g)) * u is then off by |u| |silu'(g)| dg + |silu(g)| du (plus the
       second-order terms) and by the element-wise operations: expf (2 ulp), the add, the
       fast divide (2 ulp) and the multiply; 9 ulp of |h| covers them and the oracle's own
       rounding of h to fp32.
     - s = amax / 448 differs by at most the bound of the block's largest elements plus one
       rounding, and the quotient h / s (or h * (1/s)) adds 3 ulp.
   A real mistake (a wrong code away from a tie, a dropped term) lands outside the window
   or changes many codes: at most MAX_FLIPS_PER_VECTOR flips per vector and a fraction
   MAX_FLIP_FRACTION of all compared codes are accepted.
2. y and out.  y is compared with the oracle's down projection of the GPU's own codes
   (``oracle.fp4_gemv`` on e4m3(qh) * sh), element by element within the same kind of
   a-priori bound (D * 2^-23 * sum_n |W_down[m,n] h[n]|), and within the north-star
   tolerance rel-L2 <= 1e-3, max-abs <= 1e-2 * max|ref|.  out is compared with the
   oracle's combine of those references.

Every check also reports the comparison against the oracle's own codes, with no tie rule
(``pure``), and how many codes used the tie rule.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

REL_L2 = 1e-3
MAX_ABS_FRAC = 1e-2
U23 = 2.0 ** -23                  # largest relative error of one fp32 rounding (any mode)
MAX_FLIPS_PER_VECTOR = 2
MAX_FLIP_FRACTION = 1e-4

_E4M3 = None


def e4m3_table():
    global _E4M3
    if _E4M3 is None:
        _E4M3 = np.array([oracle.e4m3_value(c) for c in range(256)])
    return _E4M3


def _sorted_values():
    tab = e4m3_table()
    return np.unique(tab[np.isfinite(tab)])  # -448 .. -0/+0 .. 448 (zeros merged)


def acc_depth(K: int) -> int:
    """Most fp32 roundings a product meets on its way into a dot product over K."""
    return 128 + K // 128 + 8


# --------------------------------------------------------------------------------- reports
def close_report(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / (nref if nref > 0 else 1.0)
    mabs = float(err.max()) if err.size else 0.0
    bound = MAX_ABS_FRAC * (float(np.abs(ref).max()) if ref.size else 0.0)
    return rel, mabs, bound


def assert_close(got, ref, what=""):
    assert np.isfinite(np.asarray(got, np.float64)).all(), f"{what}: non-finite output"
    rel, mabs, bound = close_report(got, ref)
    assert rel <= REL_L2 and mabs <= bound, \
        f"{what}: rel-L2 {rel:.3e} (<= {REL_L2}), max-abs {mabs:.3e} (<= {bound:.3e})"
    return rel, mabs


def assert_within(got, ref, bound, what=""):
    """Element-wise |got - ref| <= bound; returns the largest |got - ref| / bound."""
    got = np.asarray(got, np.float64)
    err = np.abs(got - np.asarray(ref, np.float64))
    bound = np.asarray(bound, np.float64)
    ratio = err / np.maximum(bound, 1e-300)
    worst = float(ratio.max()) if ratio.size else 0.0
    if worst > 1.0:
        i = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        raise AssertionError(f"{what}: |got - ref| = {err[i]:.3e} exceeds its bound "
                             f"{bound[i]:.3e} at {i} ({int((ratio > 1).sum())} elements)")
    return worst


# --------------------------------------------------------------------------------- inputs
def device_weights(seed, layer, E, d, f):
    import bit_moe_routed_b200 as bm
    return bm.LayerWeights.from_dict(synth.device_layer_weights(seed, layer, E, d, f))


def host_experts(seed, layer, d, f, experts):
    return {int(e): synth.host_expert(seed, layer, int(e), d, f) for e in experts}


def host_experts_q2(seed, layer, d, f, experts):
    """Routed experts in the 2-bit codec (host copies of synth's bytes), tagged for the
    oracle."""
    out = {}
    for e in experts:
        he = synth.host_expert_q2(seed, layer, int(e), d, f)
        ns = type("Q2Expert", (), {})()
        ns.__dict__.update(he.__dict__)
        ns.codec = oracle.Q2
        out[int(e)] = ns
    return out


def _gemv(codes, scales, x, codec):
    return oracle.q2_gemv(codes, scales, x) if codec == oracle.Q2 else \
        oracle.fp4_gemv(codes, scales, x)


def _abs_codes(codes, codec):
    """Codes of |W|: FP4 clears the sign bits; 2-bit codes c < 2 (the negative values)
    become 3 - c."""
    if codec != oracle.Q2:
        return codes & 0x77
    out = codes.copy()
    for i in range(4):
        neg = ((codes >> (2 * i + 1)) & 1) == 0
        out = np.where(neg, out ^ np.uint8(3 << (2 * i)), out).astype(np.uint8)
    return out


def dequant_act(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """x^ = e4m3(q) * s per 128-block, in double."""
    return e4m3_table()[q] * np.repeat(np.asarray(s, np.float64), 128, axis=-1)


# --------------------------------------------------------------------------------- bounds
def h_error_bound(ex, d: int, xhat: np.ndarray, rows):
    """A-priori bound on |h_gpu - h_oracle| for the given rows of one expert and token,
    and the exact g, u, h (double) of those rows."""
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size == 0:
        z = np.zeros(0)
        return z, z, z, z
    xabs = np.abs(xhat)
    codec = getattr(ex, "codec", oracle.FP4)
    gc, gs = ex.gate_codes[rows], ex.gate_scales[rows]
    uc, us = ex.up_codes[rows], ex.up_scales[rows]
    g = _gemv(gc, gs, xhat, codec)
    u = _gemv(uc, us, xhat, codec)
    ag = _gemv(_abs_codes(gc, codec), gs, xabs, codec)   # sum |W x|
    au = _gemv(_abs_codes(uc, codec), us, xabs, codec)
    D = acc_depth(d)
    dg, du = D * U23 * ag, D * U23 * au
    sig = 1.0 / (1.0 + np.exp(-g))
    silu = g * sig
    dsilu = sig * (1.0 + g * (1.0 - sig))
    h = silu * u
    B = 1.01 * (np.abs(u) * np.abs(dsilu) * dg + np.abs(silu) * du + 1.1 * dg * du
                + 0.25 * dg * dg * np.abs(u)) + 9 * U23 * np.abs(h)
    return B, g, u, h


def y_error_bound(down_codes, down_scales, hhat: np.ndarray, K: int,
                  codec=oracle.FP4) -> np.ndarray:
    """A-priori bound on |y_gpu - W_down h^| for an fp32 dot product over K = f."""
    return 1.01 * acc_depth(K) * U23 * _gemv(_abs_codes(down_codes, codec), down_scales,
                                             np.abs(hhat), codec)


class HStats:
    """Counts of the tie rule's use over a test."""

    def __init__(self):
        self.codes = 0
        self.flips = 0
        self.max_flips_vector = 0
        self.max_mid_rel = 0.0
        self.max_window = 0.0
        self.scales = 0
        self.scales_diff = 0
        self.max_scale_rel = 0.0

    def line(self):
        return (f"h codes: {self.flips} of {self.codes} rounded the other way at a tie "
                f"(<= {self.max_flips_vector} per vector; largest |h/s - midpoint|/|h/s| "
                f"{self.max_mid_rel:.2e}, window up to {self.max_window:.2e}); h scales: "
                f"{self.scales_diff} of {self.scales} differ (largest rel {self.max_scale_rel:.2e})")


def h_bound_from(g, u, ag, au, D):
    """The a-priori bound on |h_gpu - h| from exact g, u, sum |W x| (ag, au) and the
    depth D of the dot products (see the module docstring)."""
    dg, du = D * U23 * ag, D * U23 * au
    sig = 1.0 / (1.0 + np.exp(-g))
    silu = g * sig
    dsilu = sig * (1.0 + g * (1.0 - sig))
    h = silu * u
    return 1.01 * (np.abs(u) * np.abs(dsilu) * dg + np.abs(silu) * du + 1.1 * dg * du
                   + 0.25 * dg * dg * np.abs(u)) + 9 * U23 * np.abs(h)


def check_h_codes(qg, sg, qo, so, hf_o, ex, d, xhat, stats: HStats, what="", bound_fn=None):
    """Rule 1 for one vector (one token, one expert): GPU codes/scales (qg, sg) against the
    oracle's (qo, so, and its fp32 h before quantisation hf_o).  bound_fn(rows), if given,
    returns the h bound of those rows instead of h_error_bound(ex, d, xhat, rows)."""
    tab = e4m3_table()
    vals = _sorted_values()
    qg = np.asarray(qg, np.uint8)
    qo = np.asarray(qo, np.uint8)
    sg = np.asarray(sg, np.float32)
    so = np.asarray(so, np.float32)
    nb = qo.size // 128
    vg, vo = tab[qg], tab[qo]
    flips = np.nonzero(vg != vo)[0]
    diff_blocks = np.nonzero(sg != so)[0]
    # rows whose bound is needed: every element that differs, and in blocks whose scale
    # differs, the elements either side quantised to +-448 (the block's largest |h|)
    need = set(int(n) for n in flips)
    for b in diff_blocks:
        blk = slice(128 * b, 128 * (b + 1))
        top = np.nonzero((np.abs(vg[blk]) == 448.0) | (np.abs(vo[blk]) == 448.0))[0]
        assert top.size > 0, f"{what}: block {b} has no element at +-448"
        need |= set(int(128 * b + i) for i in top)
    rows = np.array(sorted(need), dtype=np.int64)
    B = bound_fn(rows) if bound_fn is not None else h_error_bound(ex, d, xhat, rows)[0]
    Bmap = dict(zip(rows.tolist(), B.tolist()))
    srel = np.zeros(nb)
    for b in diff_blocks:
        blk = range(128 * b, 128 * (b + 1))
        top = [n for n in blk if n in Bmap]
        amax = float(np.abs(hf_o[128 * b:128 * (b + 1)]).max())
        dmax = max(Bmap[n] for n in top)
        allowed = dmax / amax + 2 * U23
        rel = abs(float(sg[b]) - float(so[b])) / float(so[b])
        assert rel <= allowed, f"{what}: h scale of block {b} differs by {rel:.3e} " \
                               f"(derived bound {allowed:.3e})"
        srel[b] = allowed
        stats.max_scale_rel = max(stats.max_scale_rel, rel)
    for n in flips:
        b = n // 128
        i_g = np.searchsorted(vals, vg[n])
        i_o = np.searchsorted(vals, vo[n])
        assert abs(int(i_g) - int(i_o)) == 1, \
            f"{what}: h code {n} is {vg[n]} on the GPU, {vo[n]} in the oracle (not adjacent)"
        v = float(hf_o[n]) / float(so[b])
        mid = (vg[n] + vo[n]) / 2.0
        window = Bmap[int(n)] / max(abs(float(hf_o[n])), 1e-300) + srel[b] + 3 * U23
        mid_rel = abs(v - mid) / max(abs(v), 1e-300)
        assert mid_rel <= window, \
            f"{what}: h code {n} differs ({vg[n]} vs {vo[n]}) but h/s = {v!r} is " \
            f"{mid_rel:.3e} from the midpoint (derived window {window:.3e})"
        stats.max_mid_rel = max(stats.max_mid_rel, mid_rel)
        stats.max_window = max(stats.max_window, window)
    assert flips.size <= MAX_FLIPS_PER_VECTOR, \
        f"{what}: {flips.size} h codes differ from the oracle's (at most " \
        f"{MAX_FLIPS_PER_VECTOR} ties per vector)"
    stats.codes += qo.size
    stats.flips += int(flips.size)
    stats.max_flips_vector = max(stats.max_flips_vector, int(flips.size))
    stats.scales += nb
    stats.scales_diff += int(diff_blocks.size)


# --------------------------------------------------------------------------------- GPU runs
def gpu_layer(x, scores, k, weights, ws=None, keep_device=False, calls=False):
    """One layer through moe_forward (or, with calls=True, the four separate calls);
    returns every result and the intermediates left in the workspace (on the host unless
    keep_device)."""
    import bit_moe_routed_b200 as bm
    T, d = x.shape
    E, f = weights.E, weights.f
    if ws is None:
        ws = bm.alloc_workspace(T, k, E, d, f)
    run = bm.forward_calls if calls else bm.forward
    path = bm.ffn_path(T, k, weights)
    r = run(x.cuda(), scores.cuda(), k, weights, ws)
    views = bm.workspace_views(ws, T, k, E, d, f)
    if path == bm.PATH_TILES:
        views.pop("h", None)  # the tile kernels keep no fp32 h
    r.update({kk: v.clone() for kk, v in views.items()})
    if keep_device:
        return r
    bm.sync_status()
    return {kk: v.cpu() for kk, v in r.items()}


def gpu_layer_q2(x, scores, k, weights, q2, ws=None):
    """One token through moe_forward_q2 (2-bit routed experts `q2`, FP4 shared expert in
    `weights`); results and workspace intermediates on the host."""
    import bit_moe_routed_b200 as bm
    T, d = x.shape
    E, f = weights.E, weights.f
    if ws is None:
        ws = bm.alloc_workspace(T, k, E, d, f)
    r = bm.forward_q2(x.cuda(), scores.cuda(), k, weights, q2, ws)
    views = bm.workspace_views(ws, T, k, E, d, f)
    r.update({kk: v.clone() for kk, v in views.items()})
    bm.sync_status()
    return {kk: v.cpu() for kk, v in r.items()}


def check_layer(g, x, scores, k, E, d, f, seed, layer, tokens, label="", experts=None,
                verbose=True):
    """Compare GPU layer results against the oracle on the given tokens (see the module
    docstring for the rules).  Returns a summary line."""
    g = {kk: (v.cpu() if hasattr(v, "cpu") else v) for kk, v in g.items()}
    T = x.shape[0]
    P = T * k
    tokens = [int(t) for t in tokens]
    idx, w = oracle.route_topk(scores.numpy(), k)
    assert np.array_equal(g["idx"].numpy(), idx), f"{label}: routing indices differ"
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    assert np.array_equal(g["counts"].numpy(), counts), f"{label}: counts"
    assert np.array_equal(g["offsets"].numpy(), offsets), f"{label}: offsets"
    assert np.array_equal(g["perm"].numpy(), perm), f"{label}: perm"
    assert np.array_equal(g["pos"].numpy(), pos), f"{label}: pos"
    assert np.allclose(g["w"].numpy(), w, rtol=2e-6, atol=1e-7), f"{label}: gate weights"
    if experts is None:
        need = set(idx[tokens].ravel().tolist()) | {E}
        experts = host_experts(seed, layer, d, f, need)
    qx_o, sx_o = oracle.act_quant(x)
    single = T == 1 and "h" in g  # the single-token path writes qx row 0 only
    if single:
        assert np.array_equal(g["qx"].numpy()[0], qx_o[0]), f"{label}: qx (token codes)"
        assert np.array_equal(g["sx"].numpy()[0], sx_o[0]), f"{label}: sx (token scales)"
    else:
        src = np.concatenate([perm // k, np.arange(T)])
        assert np.array_equal(g["qx"].numpy(), qx_o[src]), f"{label}: qx rows"
        assert np.array_equal(g["sx"].numpy(), sx_o[src]), f"{label}: sx rows"
    qh_g, sh_g = g["qh"].numpy(), g["sh"].numpy()
    y_g, ysh_g, out_g = g["y"].numpy(), g["y_shared"].numpy(), g["out"].numpy()
    tab = e4m3_table()
    stats = HStats()
    n = len(tokens)
    y_ref = np.zeros((n, k, d))
    y_pure = np.zeros((n, k, d))
    y_bnd = np.zeros((n, k, d))
    y_got = np.zeros((n, k, d))
    ysh_ref = np.zeros((n, d))
    ysh_pure = np.zeros((n, d))
    ysh_bnd = np.zeros((n, d))
    h_worst = 0.0
    y_worst = 0.0
    for i, t in enumerate(tokens):
        xhat = dequant_act(qx_o[t], sx_o[t])
        for j in range(k + 1):
            e = int(idx[t, j]) if j < k else E
            row = int(pos[t * k + j]) if j < k else P + t
            ex = experts[e]
            yo, hq_o, hs_o, hf_o = oracle.expert_ffn_h(ex, d, f, qx_o[t:t + 1], sx_o[t:t + 1])
            what = f"{label}: token {t}, expert {e}"
            check_h_codes(qh_g[row], sh_g[row], hq_o[0], hs_o[0], hf_o[0], ex, d, xhat, stats,
                          what)
            if single:  # the fp32 h itself, against the a-priori bound, every element
                B, _, _, hx = h_error_bound(ex, d, xhat, np.arange(f))
                h_worst = max(h_worst, assert_within(g["h"].numpy()[row], hx, B,
                                                     f"{what}: fp32 h"))
            hhat = tab[qh_g[row]] * np.repeat(sh_g[row].astype(np.float64), 128)
            codec = getattr(ex, "codec", oracle.FP4)
            yr = _gemv(ex.down_codes, ex.down_scales, hhat, codec)
            yb = y_error_bound(ex.down_codes, ex.down_scales, hhat, f, codec)
            got = y_g[row] if j < k else ysh_g[t]
            y_worst = max(y_worst, assert_within(got, yr, yb, f"{what}: y"))
            if j < k:
                y_ref[i, j], y_pure[i, j], y_bnd[i, j], y_got[i, j] = yr, yo[0], yb, got
            else:
                ysh_ref[i], ysh_pure[i], ysh_bnd[i] = yr, yo[0], yb
    assert stats.flips <= max(MAX_FLIPS_PER_VECTOR, MAX_FLIP_FRACTION * stats.codes), \
        f"{label}: {stats.flips} of {stats.codes} h codes rounded the other way"
    tok = np.asarray(tokens)
    wt = w[tok]                                             # [n, k] double
    out_ref = oracle.combine(ysh_ref, y_ref, wt)
    out_pure = oracle.combine(ysh_pure, y_pure, wt)
    out_bnd = ysh_bnd + np.einsum("nk,nkd->nd", np.abs(wt), y_bnd) + \
        np.einsum("nk,nkd->nd", 2e-6 * np.abs(wt) + 1e-7, np.abs(y_ref)) + \
        (k + 2) * U23 * (np.abs(ysh_ref) + np.einsum("nk,nkd->nd", np.abs(wt), np.abs(y_ref)))
    out_worst = assert_within(out_g[tok], out_ref, out_bnd, f"{label}: out")
    ry, my = assert_close(y_got, y_ref, f"{label}: y_routed")
    rs, ms = assert_close(ysh_g[tok], ysh_ref, f"{label}: y_shared")
    ro, mo = assert_close(out_g[tok], out_ref, f"{label}: out")
    py = close_report(y_got, y_pure)
    po = close_report(out_g[tok], out_pure)
    line = (f"PARITY {label}: {n} tokens, {n * (k + 1)} (token, expert) vectors | {stats.line()}"
            f" | y vs oracle on the GPU's h codes: rel-L2 {ry:.2e}, max-abs {my:.2e}, "
            f"worst err/bound {y_worst:.2e}; y_shared rel-L2 {rs:.2e}; out rel-L2 {ro:.2e}, "
            f"worst err/bound {out_worst:.2e}" +
            (f"; fp32 h worst err/bound {h_worst:.2e}" if single else "") +
            f" | vs the oracle's own codes (no tie rule): y rel-L2 {py[0]:.2e} max-abs "
            f"{py[1]:.2e}, out rel-L2 {po[0]:.2e} max-abs {po[1]:.2e}")
    if verbose:
        print(line)
    return line


# --------------------------------------------------------------------------------- sampling
def tile_plan(counts: np.ndarray, T: int, nmax: int):
    """The FFN's token tiles of every expert (routed 0..E-1 by offsets, then the shared
    expert's T rows): list of (expert, first row, rows) in plan order."""
    E = counts.size
    offs = np.concatenate([[0], np.cumsum(counts)])
    P = int(offs[-1])
    tiles = []
    for e in range(E + 1):
        n = int(counts[e]) if e < E else T
        row = int(offs[e]) if e < E else P
        if n == 0:
            continue
        nt = -(-n // nmax)
        step = (-(-n // nt) + 15) // 16 * 16
        for i in range(nt):
            tiles.append((e, row + i * step, min(step, n - i * step)))
    return tiles


def tile_sample_tokens(idx: np.ndarray, E: int, n: int = 64, seed: int = 0):
    """Tokens to check in a large batch, chosen to cover the tile kernels' edges: the
    hottest expert's last tile, the last row of the last tile of the highest experts in
    plan order (the tail the stream-K split cuts), the last row of the first tile of
    experts with several tiles, the first and last tokens (the shared expert's first and
    last tile), then seeded random tokens up to n."""
    T, k = idx.shape
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    nmax = 32 if T <= 64 else 112
    tiles = tile_plan(counts, T, nmax)
    pick = []

    def add_row(r):
        t = int(perm[r]) // k if r < T * k else r - T * k
        if t not in pick and len(pick) < n:
            pick.append(t)

    add_row(T * k)           # token 0 in the shared expert's first tile
    add_row(T * k + T - 1)   # the last token: the shared expert's last tile, last row
    hot = int(np.argmax(counts))
    last = [tl for tl in tiles if tl[0] == hot][-1]
    for r in range(last[1] + last[2] - 1, last[1] - 1, -1)[:16]:
        add_row(r)
    routed = [tl for tl in tiles if tl[0] < E]
    ends = {}
    for e, r0, m in routed:
        ends[e] = r0 + m - 1
    for e in sorted(ends)[::-1][:16]:
        add_row(ends[e])
    firsts = {}
    for e, r0, m in routed:
        if e not in firsts and int(counts[e]) > nmax:
            firsts[e] = r0 + m - 1
    for e in sorted(firsts)[:8]:
        add_row(firsts[e])
    rng = np.random.default_rng(seed)
    for t in rng.permutation(T):
        if len(pick) >= n:
            break
        if int(t) not in pick:
            pick.append(int(t))
    return sorted(pick)
