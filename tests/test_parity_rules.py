"""CPU checks of the comparison rule the GPU parity tests use for the e4m3
re-quantisation of h: an element exactly on a rounding tie gets an allowance equal to
the effect of rounding it the other way, and elements away from ties get none."""
import numpy as np

import oracle
import synth
from helpers import TIE_REL, tie_allowance


def test_allowance_equals_effect_of_the_other_rounding():
    d, f = 256, 128
    ex = synth.host_expert(7, 0, 2, d, f)
    rng = np.random.default_rng(0)
    hf = rng.normal(0, 1, f).astype(np.float32)
    hf[0] = 8.0                                   # block max: s = 8/448 exactly
    s = np.float32(8.0) / np.float32(448.0)
    hf[5] = np.float32(6.25 * s)                  # 6.25 = midpoint of e4m3 6.0 and 6.5
    q, sc = oracle.quant_blocks(hf)
    v5 = np.float32(hf[5]) / sc[0]
    assert abs(v5 - 6.25) / 6.25 < TIE_REL
    allow = tie_allowance(ex, q, sc, hf)
    hh = np.array([oracle.e4m3_value(int(c)) for c in q]) * float(sc[0])
    alt = hh.copy()
    other = 6.5 if abs(hh[5]) / sc[0] == 6.0 else 6.0
    alt[5] = np.sign(hh[5]) * other * float(sc[0])
    ya = oracle.fp4_gemv(ex.down_codes, ex.down_scales, hh)
    yb = oracle.fp4_gemv(ex.down_codes, ex.down_scales, alt)
    assert np.all(np.abs(ya - yb) <= allow * (1 + 1e-12) + 1e-12)
    assert np.allclose(allow, np.abs(ya - yb), rtol=1e-12, atol=1e-12)


def test_no_allowance_away_from_ties():
    d, f = 256, 128
    ex = synth.host_expert(7, 0, 3, d, f)
    hf = np.linspace(-3, 3, f).astype(np.float32)
    q, sc = oracle.quant_blocks(hf)
    tab = np.array([oracle.e4m3_value(c) for c in range(256)])
    mags = np.unique(np.abs(tab[np.isfinite(tab)]))
    mids = (mags[1:] + mags[:-1]) / 2
    v = np.abs(hf / sc[0]).astype(np.float64)
    near = np.min(np.abs(v[:, None] - mids[None, :]) / np.maximum(v[:, None], 1e-30), axis=1)
    allow = tie_allowance(ex, q, sc, hf)
    if (near > TIE_REL).all():
        assert not allow.any()
