"""Pins for the oracle's FP8 weight codec and fp8_gemm (CPU only).

- fp8_gemm against a float64 numpy matmul of operands decoded by torch's float8_e4m3fn
  (a library routine) and scaled per 128-block / 128 x 128 block, on inputs chosen so that
  every partial sum is exact in float64 (then any summation order gives the same bits):
  a wrong scale index, a transposed operand or a dropped term fails it.
- An FP4 expert whose ue8m0 scales are constant over 128 x 128 blocks is also an FP8
  expert (every e2m1 value is an e4m3 value, the scale a power of two), so its FFN through
  the FP8 codec must equal its FFN through the FP4 codec bit for bit; the FP4 path is
  pinned against a dense float64 FFN (test_oracle_ffn.py).
"""
import numpy as np
import pytest
import torch

import oracle

E2M1_TO_E4M3 = {}


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def exact_codes(rng, shape):
    """e4m3 codes with exponents in a narrow band (|v| in [2^-3, 15]), either sign."""
    exp = rng.integers(4, 11, shape)          # biased exponent 4..10 -> 2^-3 .. 2^3
    man = rng.integers(0, 8, shape)
    sign = rng.integers(0, 2, shape)
    return ((sign << 7) | (exp << 3) | man).astype(np.uint8)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (3, 256, 384), (8, 384, 256)])
def test_fp8_gemm_against_exact_float64_matmul(M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    A = exact_codes(rng, (M, K))
    B = exact_codes(rng, (N, K))
    sa = (2.0 ** rng.integers(-4, 5, (M, K // 128))).astype(np.float32)
    sb = (2.0 ** rng.integers(-4, 5, (N // 128, K // 128))).astype(np.float32)
    a = e4m3_values(A) * np.repeat(sa.astype(np.float64), 128, axis=1)
    b = e4m3_values(B) * np.repeat(np.repeat(sb.astype(np.float64), 128, axis=0), 128, axis=1)
    want = a @ b.T
    got = oracle.fp8_gemm(A, sa, B, sb)
    assert np.array_equal(got, want)
    assert np.abs(want).max() > 0


def test_fp8_gemm_block_scale_indexing():
    """One nonzero weight per 128 x 128 block: C picks up exactly that block's scale."""
    M, N, K = 1, 256, 256
    A = np.full((M, K), 0x38, np.uint8)  # 1.0
    B = np.zeros((N, K), np.uint8)
    B[0, 0] = 0x38
    B[0, 200] = 0x40          # 2.0 in block (0, 1)
    B[130, 5] = 0x38          # block (1, 0)
    sa = np.array([[1.0, 0.5]], np.float32)
    sb = np.array([[2.0, 4.0], [8.0, 16.0]], np.float32)
    C = oracle.fp8_gemm(A, sa, B, sb)
    assert C[0, 0] == 1.0 * 2.0 + 2.0 * 0.5 * 4.0
    assert C[0, 130] == 1.0 * 8.0
    assert C[0, 1] == 0.0


E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e2m1_to_e4m3(nib: np.ndarray) -> np.ndarray:
    vals = np.array([E2M1[n & 7] * (-1 if n & 8 else 1) for n in range(16)])
    enc = {}
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        enc.setdefault(float(e4m3_values(np.array([c]))[0]), c)
    enc[-0.0] = 0x80
    table = np.array([enc[float(v)] if not (v == 0 and n & 8) else 0x80
                      for n, v in enumerate(vals)], np.uint8)
    return table[nib]


class _Ex:
    def __init__(self, codec, **kw):
        self.codec = codec
        self.__dict__.update(kw)


def block_scaled_fp4(rng, rows, K):
    """FP4 codes with ue8m0 scales constant over 128 x 128 blocks; the same matrix as FP8."""
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    blk = rng.integers(120, 126, (rows // 128, K // 128)).astype(np.uint8)
    scales = np.repeat(np.repeat(blk, 128, axis=0), 4, axis=1)  # per 32 along K
    nib = np.stack([codes & 0x0F, codes >> 4], axis=-1).reshape(rows, K)
    f8 = e2m1_to_e4m3(nib)
    s8 = (2.0 ** (blk.astype(np.float64) - 127)).astype(np.float32)
    return (codes, scales), (f8, s8)


def test_fp8_expert_equals_its_fp4_twin():
    rng = np.random.default_rng(21)
    d, f, ntok = 256, 256, 2
    mats4, mats8 = {}, {}
    for m, (rows, K) in (("gate", (f, d)), ("up", (f, d)), ("down", (d, f))):
        (c4, s4), (c8, s8) = block_scaled_fp4(rng, rows, K)
        mats4[f"{m}_codes"], mats4[f"{m}_scales"] = c4, s4
        mats8[f"{m}_codes"], mats8[f"{m}_scales"] = c8, s8
    x = rng.standard_normal((ntok, d)).astype(np.float32)
    qx, sx = oracle.quant_blocks(x.ravel())
    qx, sx = qx.reshape(ntok, d), sx.reshape(ntok, d // 128)
    y4, hq4, hs4 = oracle.expert_ffn(_Ex(oracle.FP4, **mats4), d, f, qx, sx, want_h=True)
    y8, hq8, hs8 = oracle.expert_ffn(_Ex(oracle.FP8, **mats8), d, f, qx, sx, want_h=True)
    assert np.array_equal(y4, y8)
    assert np.array_equal(hq4, hq8) and np.array_equal(hs4, hs8)
    assert np.abs(y4).max() > 0
