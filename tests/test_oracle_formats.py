"""Pins for the oracle's number formats and quantiser (CPU only).

The oracle's tables and its e4m3 encoder are checked against things other than
itself: the OCP MX / OFP8 format definitions (golden files), torch's float8
decoders and casts (library routines), and brute-force nearest search.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLD, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            rows.append((int(c), float(v)))
    return rows


def test_e2m1_table_matches_ocp_values():
    rows = _golden("e2m1_values.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1_value(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def test_e4m3_table_matches_torch_decoder_all_codes():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        got = oracle.e4m3_value(c)
        r = float(ref[c])
        if math.isnan(r):
            assert math.isnan(got), c
        else:
            assert got == r and math.copysign(1, got) == math.copysign(1, r), (c, got, r)


def test_e4m3_landmarks():
    for code, val in _golden("e4m3_landmarks.txt"):
        assert oracle.e4m3_value(code) == val
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))


def test_ue8m0_table_matches_torch_decoder_all_codes():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64)
    for c in range(256):
        got = oracle.ue8m0_value(c)
        r = float(ref[c])
        assert (math.isnan(got) and math.isnan(r)) or got == r, (c, got, r)


def _finite_e4m3():
    codes = [c for c in range(256) if not math.isnan(oracle.e4m3_value(c))]
    vals = np.array([oracle.e4m3_value(c) for c in codes])
    return np.array(codes), vals


def _brute_force_encode(v: float) -> int:
    """Nearest finite e4m3 value; ties to the even mantissa; |v| > 448 saturates."""
    codes, vals = _finite_e4m3()
    if v > 448:
        return 0x7E
    if v < -448:
        return 0xFE
    dist = np.abs(vals - v)
    best = dist.min()
    cand = [int(c) for c, dd in zip(codes, dist) if dd == best]
    # zero of the same sign as v
    if best == abs(v) and any(oracle.e4m3_value(c) == 0 for c in cand):
        return 0x80 if (v < 0 or (v == 0 and math.copysign(1, v) < 0)) else 0x00
    if len(cand) == 1:
        return cand[0]
    even = [c for c in cand if (c & 1) == 0]
    assert len(even) == 1, (v, cand)
    return even[0]


def test_e4m3_encode_brute_force_on_values_and_midpoints():
    _, vals = _finite_e4m3()
    pos = np.unique(vals[vals >= 0])
    mids = (pos[1:] + pos[:-1]) / 2
    probes = np.concatenate([pos, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
                             np.nextafter(mids.astype(np.float32), np.float32(1000)),
                             [448.0, 455.0, 463.9, 464.0, 470.0, 1e6, 2.0 ** -10, 2.0 ** -11,
                              0.9 * 2.0 ** -10, 1.1 * 2.0 ** -10]]).astype(np.float32)
    probes = np.concatenate([probes, -probes])
    got = oracle.e4m3_encode(probes)
    for v, g in zip(probes, got):
        assert int(g) == _brute_force_encode(float(v)), (float(v), int(g))


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 100, 20000),
                        rng.uniform(-2 ** -6, 2 ** -6, 5000), rng.uniform(-463, 463, 5000)])
    v = v.astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(v)
    assert np.array_equal(got, ref)


def test_quant_blocks_against_torch_cast():
    rng = np.random.default_rng(2)
    v = rng.normal(0, 1, 128 * 16).astype(np.float32)
    q, s = oracle.quant_blocks(v)
    vt = torch.from_numpy(v).view(16, 128)
    st = vt.abs().amax(dim=1) / torch.tensor(448.0, dtype=torch.float32)
    assert np.array_equal(s, st.numpy())
    qt = (vt / st[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy().ravel()
    assert np.array_equal(q, qt)


def test_quant_blocks_special_cases():
    # a block holding 448 has scale exactly 1 and e4m3-representable values are exact
    _, vals = _finite_e4m3()
    rep = vals[(vals <= 448) & (vals >= -448)]
    rng = np.random.default_rng(3)
    blk = rng.choice(rep, 128).astype(np.float32)
    blk[5] = 448.0
    q, s = oracle.quant_blocks(blk)
    assert s[0] == 1.0
    assert np.array_equal(np.array([oracle.e4m3_value(int(c)) for c in q]), blk.astype(np.float64))
    # all-zero block: scale 1, codes 0
    q, s = oracle.quant_blocks(np.zeros(128, np.float32))
    assert s[0] == 1.0 and not q.any()
    # the block maximum always maps to code +-448
    v = rng.normal(0, 3, 128).astype(np.float32)
    q, s = oracle.quant_blocks(v)
    i = int(np.argmax(np.abs(v)))
    assert oracle.e4m3_value(int(q[i])) == math.copysign(448.0, v[i])


def test_act_quant_bf16_rows():
    rng = np.random.default_rng(4)
    x = torch.from_numpy(rng.normal(0, 1, (3, 512)).astype(np.float32)).to(torch.bfloat16)
    q, s = oracle.act_quant(x)
    xf = x.to(torch.float32).view(3, 4, 128)
    st = xf.abs().amax(dim=2) / torch.tensor(448.0)
    qt = (xf / st[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(3, 512).numpy()
    assert np.array_equal(s, st.numpy()) and np.array_equal(q, qt)
