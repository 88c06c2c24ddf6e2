"""Pins for the oracle's 2-bit routed-expert codec (CPU only).

- The value table against the golden file (the codec's reading), and the bit rate the
  page prints (2.0625 bits per weight) from the array sizes.
- The 2-bit GEMV against int64 numpy sums on integer-exact inputs, with the codes
  unpacked by numpy (a wrong bit order, element order or scale index fails it).
- Every 2-bit weight (+-0.5, +-1.5 times a power of two) is also an FP4 weight, so a
  2-bit expert re-encoded as FP4 (e2m1 codes, its per-128 scale repeated per 32) must give
  the same FFN output bit for bit through the FP4 path, which is itself pinned against a
  dense float64 FFN (test_oracle_ffn.py); the same holds for a whole layer with 2-bit
  routed experts and an FP4 shared expert.
"""
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _q2_table():
    vals = {}
    with open(os.path.join(GOLD, "q2_values.txt")) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                vals[int(c)] = float(v)
    return vals


Q2 = _q2_table()


def unpack(codes):
    """[rows, K/4] bytes -> [rows, K] 2-bit codes, element 4i + j in bits 2j..2j+1."""
    rows = codes.shape[0]
    return np.stack([(codes >> (2 * j)) & 3 for j in range(4)], axis=-1).reshape(rows, -1)


def test_value_table_and_bit_rate():
    assert sorted(Q2) == [0, 1, 2, 3]
    for c, v in Q2.items():
        assert oracle.q2_value(c) == v
    rows, K = 2048, 4096
    bits = 8 * (rows * K // 4 + rows * K // 128) / (rows * K)
    assert bits == 2.0625


def test_q2_gemv_against_int64_numpy():
    rng = np.random.default_rng(11)
    rows, K = 24, 512
    codes = rng.integers(0, 256, (rows, K // 4), dtype=np.uint8)
    scales = rng.integers(124, 131, (rows, K // 128), dtype=np.uint8)  # 2^-3 .. 2^3
    xi = rng.integers(-64, 65, K).astype(np.int64)  # xhat = xi * 2^-6
    xhat = xi * 2.0 ** -6
    got = oracle.q2_gemv(codes, scales, xhat)
    # w = (2c - 3) / 2 * 2^(s - 127); sum in integers with the common factor 2^-(1+6+3+...)
    c2 = 2 * unpack(codes).astype(np.int64) - 3
    sexp = np.repeat(scales.astype(np.int64) - 127, 128, axis=1)  # [rows, K]
    lo = sexp.min()
    num = (c2 * (np.int64(1) << (sexp - lo)) * xi[None, :]).sum(axis=1)
    want = num.astype(np.float64) * 2.0 ** (lo - 1 - 6)
    assert np.array_equal(got, want)


def test_q2_element_order_and_scale_index():
    rows, K = 1, 256
    codes = np.zeros((rows, K // 4), np.uint8)
    codes[0, 5] = 0b11_10_01_00  # elements 20..23 -> codes 0, 1, 2, 3
    scales = np.array([[127, 129]], np.uint8)  # 1 for elements 0..127, 4 for 128..255
    for el, want in ((20, -1.5), (21, -0.5), (22, 0.5), (23, 1.5), (0, -1.5), (200, -6.0)):
        x = np.zeros(K)
        x[el] = 1.0
        assert oracle.q2_gemv(codes, scales, x)[0] == want, el


E2M1_CODE = {-1.5: 0b1011, -0.5: 0b1001, 0.5: 0b0001, 1.5: 0b0011}


def q2_as_fp4(codes, scales):
    """The same matrix in FP4: e2m1 codes of +-0.5 / +-1.5, each per-128 scale repeated
    for its four 32-blocks."""
    c = unpack(codes)
    vals = np.vectorize(lambda v: Q2[v])(c)
    nib = np.vectorize(lambda v: E2M1_CODE[v])(vals).astype(np.uint8)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return packed, np.repeat(scales, 4, axis=1)


class _Ex:
    def __init__(self, codec, **kw):
        self.codec = codec
        self.__dict__.update(kw)


def q2_expert(rng, d, f):
    mk = lambda rows, K: (rng.integers(0, 256, (rows, K // 4), dtype=np.uint8),  # noqa: E731
                          rng.integers(120, 125, (rows, K // 128), dtype=np.uint8))
    gc, gs = mk(f, d)
    uc, us = mk(f, d)
    dc, ds = mk(d, f)
    return _Ex(oracle.Q2, gate_codes=gc, gate_scales=gs, up_codes=uc, up_scales=us,
               down_codes=dc, down_scales=ds)


def as_fp4(ex):
    out = {}
    for m in ("gate", "up", "down"):
        c, s = q2_as_fp4(getattr(ex, f"{m}_codes"), getattr(ex, f"{m}_scales"))
        out[f"{m}_codes"], out[f"{m}_scales"] = c, s
    return _Ex(oracle.FP4, **out)


def test_q2_expert_equals_its_fp4_encoding():
    rng = np.random.default_rng(12)
    d, f, ntok = 256, 256, 3
    ex = q2_expert(rng, d, f)
    x = rng.standard_normal((ntok, d)).astype(np.float32)
    qx, sx = oracle.quant_blocks(x.ravel())
    qx, sx = qx.reshape(ntok, d), sx.reshape(ntok, d // 128)
    y2, hq2, hs2 = oracle.expert_ffn(ex, d, f, qx, sx, want_h=True)
    y4, hq4, hs4 = oracle.expert_ffn(as_fp4(ex), d, f, qx, sx, want_h=True)
    assert np.array_equal(y2, y4)
    assert np.array_equal(hq2, hq4) and np.array_equal(hs2, hs4)
    assert np.abs(y2).max() > 0


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (3, 6, 3)])
def test_layer_with_q2_routed_experts_equals_fp4_encoding(T, E, k):
    import torch
    rng = np.random.default_rng(13 + T)
    d, f = 256, 128
    routed = {e: q2_expert(rng, d, f) for e in range(E)}
    shared = as_fp4(q2_expert(rng, d, f))  # an FP4 shared expert
    x = torch.randn(T, d).to(torch.bfloat16)
    scores = rng.random((T, E)).astype(np.float32)
    idx, w = oracle.route_topk(scores, k)
    mixed = dict(routed)
    mixed[E] = shared
    all_fp4 = {e: as_fp4(ex) for e, ex in routed.items()}
    all_fp4[E] = shared
    a = oracle.moe_layer(x, E, k, d, f, mixed, idx, w)
    b = oracle.moe_layer(x, E, k, d, f, all_fp4, idx, w)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
