"""CPU checks of the comparison rules the GPU parity tests use (see helpers.py):

- the a-priori bound on the fp32 hidden state covers an fp32 emulation of the blocked
  dot products (products exact, fp32 sums per 128-element chunk, one fused scale-and-add
  per chunk) and of the element-wise SwiGLU;
- a code that rounds the other way at a tie is accepted and counted, while a code changed
  away from a tie, a change by two code steps, a scale off by more than its bound, or too
  many flips in one vector are caught;
- the element-wise bound on y catches a wrong down projection.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import (HStats, U23, acc_depth, check_h_codes, dequant_act, e4m3_table,
                     h_error_bound, y_error_bound, assert_within)

D, F = 1024, 256


@pytest.fixture(scope="module")
def case():
    ex = synth.host_expert(7, 0, 2, D, F)
    x = synth.gen_x(1, D, seed=11)
    qx, sx = oracle.act_quant(x)
    y, hq, hs, hf = oracle.expert_ffn_h(ex, D, F, qx, sx)
    return ex, qx, sx, dequant_act(qx[0], sx[0]), hq[0], hs[0], hf[0]


def _fp32_blocked_dot(codes, scales, q, s):
    """fp32 emulation: per 128-chunk a sequential fp32 sum of exact products, then one
    fused multiply-add by the chunk's activation scale into the fp32 total."""
    tab2 = np.array([oracle.e2m1_value(c) for c in range(16)])
    rows, K = codes.shape[0], codes.shape[1] * 2
    w = np.empty((rows, K))
    w[:, 0::2] = tab2[codes & 15]
    w[:, 1::2] = tab2[codes >> 4]
    w *= np.exp2(np.repeat(scales.astype(np.float64) - 127.0, 32, axis=1))
    xq = e4m3_table()[q]
    out = np.zeros(rows, np.float32)
    for c in range(K // 128):
        prod = (w[:, 128 * c:128 * (c + 1)] * xq[128 * c:128 * (c + 1)]).astype(np.float32)
        part = np.zeros(rows, np.float32)
        for i in range(128):
            part = (part + prod[:, i]).astype(np.float32)
        out = np.float32(np.float64(out) + np.float64(s[c]) * np.float64(part))
    return out


def test_h_bound_covers_fp32_arithmetic(case):
    ex, qx, sx, xhat, hq, hs, hf = case
    g32 = _fp32_blocked_dot(ex.gate_codes, ex.gate_scales, qx[0], sx[0])
    u32 = _fp32_blocked_dot(ex.up_codes, ex.up_scales, qx[0], sx[0])
    e = np.exp(-g32.astype(np.float64)).astype(np.float32)
    h32 = (g32 / (np.float32(1) + e)).astype(np.float32) * u32
    B, g, u, h = h_error_bound(ex, D, xhat, np.arange(F))
    assert np.all(np.abs(h32.astype(np.float64) - h) <= B)
    assert np.all(np.abs(hf.astype(np.float64) - h) <= B)  # the oracle's own fp32 h
    # the bound is a worst case: far above the observed error, far below |h|
    assert np.median(B / np.maximum(np.abs(h), 1e-30)) < 2e-3


def test_depth_counts_the_blocked_structure():
    assert acc_depth(4096) == 128 + 32 + 8
    assert acc_depth(2048) == 128 + 16 + 8


def _nearest_tie(hf, hs):
    tab = e4m3_table()
    mags = np.unique(np.abs(tab[np.isfinite(tab)]))
    v = np.abs(hf.astype(np.float64) / np.repeat(hs.astype(np.float64), 128))
    i = np.clip(np.searchsorted(mags, v), 1, len(mags) - 1)
    mid = (mags[i - 1] + mags[i]) / 2
    dist = np.abs(v - mid) / np.maximum(v, 1e-30)
    dist[v >= 448] = np.inf
    return dist


def _flip(q, n, steps=1):
    """The code `steps` values away from q[n] toward the other side of its rounding."""
    tab = e4m3_table()
    vals = np.unique(tab[np.isfinite(tab)])
    q = q.copy()
    i = int(np.searchsorted(vals, tab[q[n]]))
    target = vals[i + steps] if i + steps < len(vals) else vals[i - steps]
    q[n] = int(np.nonzero(tab == target)[0][0])
    return q


def test_flip_at_a_tie_is_accepted_and_counted(case):
    ex, qx, sx, xhat, hq, hs, hf = case
    dist = _nearest_tie(hf, hs)
    n = int(np.argmin(dist))
    tab = e4m3_table()
    v = hf[n] / hs[n // 128]
    # flip toward the midpoint's other side
    vals = np.unique(tab[np.isfinite(tab)])
    i = int(np.searchsorted(vals, tab[hq[n]]))
    other = vals[i + 1] if v > tab[hq[n]] else vals[i - 1]
    q = hq.copy()
    q[n] = int(np.nonzero(tab == other)[0][0])
    st = HStats()
    check_h_codes(q, hs, hq, hs, hf, ex, D, xhat, st, "tie")
    assert st.flips == 1 and st.codes == F


def test_flip_away_from_a_tie_is_caught(case):
    ex, qx, sx, xhat, hq, hs, hf = case
    dist = _nearest_tie(hf, hs)
    n = int(np.argmax(np.where(np.isfinite(dist), dist, -1)))
    assert dist[n] > 1e-2
    with pytest.raises(AssertionError, match="from the midpoint"):
        check_h_codes(_flip(hq, n), hs, hq, hs, hf, ex, D, xhat, HStats(), "far")


def test_two_step_change_is_caught(case):
    ex, qx, sx, xhat, hq, hs, hf = case
    n = int(np.argmin(_nearest_tie(hf, hs)))
    with pytest.raises(AssertionError, match="not adjacent"):
        check_h_codes(_flip(hq, n, 2), hs, hq, hs, hf, ex, D, xhat, HStats(), "two steps")


def test_wrong_scale_is_caught(case):
    ex, qx, sx, xhat, hq, hs, hf = case
    s = hs.copy()
    s[0] = np.float32(s[0] * np.float32(1.001))
    with pytest.raises(AssertionError, match="scale of block 0"):
        check_h_codes(hq, s, hq, hs, hf, ex, D, xhat, HStats(), "scale")


def test_too_many_flips_in_one_vector_are_caught(case, monkeypatch):
    ex, qx, sx, xhat, hq, hs, hf = case
    import helpers
    order = np.argsort(_nearest_tie(hf, hs))[:3]
    q = hq.copy()
    tab = e4m3_table()
    vals = np.unique(tab[np.isfinite(tab)])
    for n in order:
        v = hf[n] / hs[n // 128]
        i = int(np.searchsorted(vals, tab[q[n]]))
        other = vals[i + 1] if v > tab[q[n]] else vals[i - 1]
        q[n] = int(np.nonzero(tab == other)[0][0])
    # the three nearest ties may lie outside the window; widen it so only the count decides
    monkeypatch.setattr(helpers, "acc_depth", lambda K: 10 ** 6)
    with pytest.raises(AssertionError, match="ties per vector"):
        check_h_codes(q, hs, hq, hs, hf, ex, D, xhat, HStats(), "count")


def test_y_bound_catches_a_wrong_down_projection(case):
    ex, qx, sx, xhat, hq, hs, hf = case
    hhat = dequant_act(hq, hs)
    y = oracle.fp4_gemv(ex.down_codes, ex.down_scales, hhat)
    yb = y_error_bound(ex.down_codes, ex.down_scales, hhat, F)
    # an fp32 rounding of every element passes; an error of 1e-4 relative does not
    y32 = y.astype(np.float32)
    assert assert_within(y32, y, yb) <= 1.0
    bad = y.copy()
    bad[5] += 1e-4 * np.abs(y).max()
    with pytest.raises(AssertionError, match="exceeds its bound"):
        assert_within(bad, y, yb, "y")
    assert np.all(yb < 1e-4 * np.abs(y).max())
    assert np.all(yb > 0)
    assert U23 == 2.0 ** -23
