"""Shared helpers for the parity tests: seeded inputs for both sides, oracle references,
and the comparison rules.

Integers and codes (routing indices, dispatch permutation, activation codes and scales)
must match bit-exactly.  Floating-point layer outputs must be within rel-L2 <= 1e-3 and
max-abs <= 1e-2 * max|ref| of the oracle, with one allowance that the method itself
makes necessary.

The hidden state h = silu(g) * u is re-quantised to e4m3 (3 mantissa bits) from fp32.
The oracle sums g and u in double and the GPU in fp32, so their fp32 h can differ by a
few 1e-7 relative.  An element whose h / s lies within TIE_REL of an e4m3 rounding
midpoint may therefore round either way on a correct implementation: both codes are
valid results.  For those elements only, the comparison allows the exact effect of the
other rounding, |W_down[:, n]| * |code step| * s, propagated through the combine.
Measured on a B200, GPU and oracle h codes differ in about 1 of 10^5 elements, always
within 6e-7 of a midpoint; TIE_REL = 4e-6 leaves about 8x headroom and marks about
0.1 element per (token, expert) pair.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

REL_L2 = 1e-3
MAX_ABS_FRAC = 1e-2
TIE_REL = 4e-6

_E4M3 = None


def _e4m3_table():
    global _E4M3
    if _E4M3 is None:
        _E4M3 = np.array([oracle.e4m3_value(c) for c in range(256)])
    return _E4M3


def close_report(got, ref, allow=None):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    if allow is not None:
        err = np.maximum(0.0, err - np.asarray(allow, np.float64))
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / (nref if nref > 0 else 1.0)
    mabs = float(err.max()) if err.size else 0.0
    bound = MAX_ABS_FRAC * (float(np.abs(ref).max()) if ref.size else 0.0)
    return rel, mabs, bound


def assert_close(got, ref, what="", allow=None):
    assert np.isfinite(np.asarray(got, np.float64)).all(), f"{what}: non-finite output"
    rel, mabs, bound = close_report(got, ref, allow)
    assert rel <= REL_L2 and mabs <= bound, \
        f"{what}: rel-L2 {rel:.3e} (<= {REL_L2}), max-abs {mabs:.3e} (<= {bound:.3e})"


def device_weights(seed, layer, E, d, f):
    import bit_moe_routed_b200 as bm
    return bm.LayerWeights.from_dict(synth.device_layer_weights(seed, layer, E, d, f))


def host_experts(seed, layer, d, f, experts):
    return {int(e): synth.host_expert(seed, layer, int(e), d, f) for e in experts}


def _down_column(ex, n: int) -> np.ndarray:
    """Column n of the dequantised down matrix [d] (codes [d][f/2], scales [d][f/32])."""
    byte = ex.down_codes[:, n // 2]
    code = (byte >> 4) if (n & 1) else (byte & 0x0F)
    e = (code >> 1) & 3
    m = code & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + m / 2.0, e - 1))
    val = np.where(code & 8, -mag, mag)
    return val * np.exp2(ex.down_scales[:, n // 32].astype(np.float64) - 127.0)


def tie_allowance(ex, hq, hs, hf) -> np.ndarray:
    """Bound on |y| change if any near-tie element of h rounds the other way [d]."""
    tab = _e4m3_table()
    mags = np.unique(np.abs(tab[np.isfinite(tab)]))
    s = np.repeat(hs.astype(np.float64), 128)
    a = np.abs(hf.astype(np.float64) / s)
    i = np.clip(np.searchsorted(mags, a), 1, len(mags) - 1)
    lo, hi = mags[i - 1], mags[i]
    mid = (lo + hi) / 2
    tie = (a < 448.0) & (np.abs(a - mid) <= TIE_REL * np.maximum(a, 1e-30))
    allow = np.zeros(ex.down_codes.shape[0])
    for n in np.nonzero(tie)[0]:
        allow += np.abs(_down_column(ex, int(n))) * (hi[n] - lo[n]) * s[n]
    return allow


def oracle_pairs(x, scores, k, E, d, f, experts, tokens):
    """Oracle per selected token: routing, y per routed pair, y_sh, out, and the tie
    allowances of each, all from the oracle's own computation."""
    idx, w = oracle.route_topk(scores.numpy(), k)
    qx, sx = oracle.act_quant(x[torch.as_tensor(tokens)])
    n = len(tokens)
    y = np.zeros((n, k, d))
    ysh = np.zeros((n, d))
    ay = np.zeros((n, k, d))
    ash = np.zeros((n, d))
    out = np.zeros((n, d))
    aout = np.zeros((n, d))
    for i, t in enumerate(tokens):
        for j in range(k + 1):
            e = int(idx[t, j]) if j < k else E
            yy, hq, hs, hf = oracle.expert_ffn_h(experts[e], d, f, qx[i:i + 1], sx[i:i + 1])
            al = tie_allowance(experts[e], hq[0], hs[0], hf[0])
            if j < k:
                y[i, j], ay[i, j] = yy[0], al
            else:
                ysh[i], ash[i] = yy[0], al
        out[i] = oracle.combine(ysh[i:i + 1], y[i:i + 1], w[t:t + 1])[0]
        aout[i] = ash[i] + np.abs(w[t]) @ ay[i]
    return idx, w, y, ysh, out, ay, ash, aout


def gpu_layer(x, scores, k, weights, ws=None):
    import bit_moe_routed_b200 as bm
    r = bm.forward(x.cuda(), scores.cuda(), k, weights, ws)
    bm.sync_status()
    return {kk: v.cpu() for kk, v in r.items()}


def check_layer(g, x, scores, k, E, d, f, seed, layer, tokens, label="", experts=None):
    """Compare GPU layer results against the oracle on the given tokens."""
    idx_all, _ = oracle.route_topk(scores.numpy(), k)
    if experts is None:
        need = set(idx_all[tokens].ravel().tolist()) | {E}
        experts = host_experts(seed, layer, d, f, need)
    idx, w, y_pair, y_sh, out, ay, ash, aout = oracle_pairs(x, scores, k, E, d, f, experts,
                                                            tokens)
    assert np.array_equal(g["idx"].numpy(), idx), f"{label}: routing indices differ"
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    assert np.array_equal(g["counts"].numpy(), counts), f"{label}: counts"
    assert np.array_equal(g["offsets"].numpy(), offsets), f"{label}: offsets"
    assert np.array_equal(g["perm"].numpy(), perm), f"{label}: perm"
    assert np.array_equal(g["pos"].numpy(), pos), f"{label}: pos"
    assert np.allclose(g["w"].numpy(), w, rtol=2e-6, atol=1e-7), f"{label}: gate weights"
    tok = np.asarray(tokens)
    y_gpu = g["y"].numpy()[pos.reshape(-1, k)[tok]]  # [n, k, d]
    assert_close(y_gpu, y_pair, f"{label}: y_routed", ay)
    assert_close(g["y_shared"].numpy()[tok], y_sh, f"{label}: y_shared", ash)
    assert_close(g["out"].numpy()[tok], out, f"{label}: out", aout)
