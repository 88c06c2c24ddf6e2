"""Pins for the oracle's FP4 GEMV, expert FFN, combine and whole layer (CPU only).

References used: int64 numpy sums on integer-exact inputs, a dense float64 FFN
assembled from library routines (numpy matmul, torch's e4m3 cast) over weights
dequantised with the OCP e2m1 values, and invariants of the method (token
permutation, k = 1 with weight 1, Σw = 1).
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _e2m1_table():
    vals = np.zeros(16)
    with open(os.path.join(GOLD, "e2m1_values.txt")) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                c, v = line.split()
                vals[int(c)] = float(v)
    return vals


E2M1 = _e2m1_table()


def _nibbles(codes):
    """[rows, K/2] bytes -> [rows, K] 4-bit codes, element 2i in the low nibble."""
    rows = codes.shape[0]
    return np.stack([codes & 0x0F, codes >> 4], axis=-1).reshape(rows, -1)


def dense(codes, scales):
    c = _nibbles(codes)
    sc = np.exp2(scales.astype(np.float64) - 127.0).repeat(32, axis=1)
    return E2M1[c] * sc


def torch_quant(v32: torch.Tensor):
    """Per-128 e4m3 quantisation with torch's cast; returns the dequantised float64."""
    n = v32.shape[-1]
    b = v32.reshape(*v32.shape[:-1], n // 128, 128)
    s = b.abs().amax(dim=-1) / torch.tensor(448.0)
    s = torch.where(s == 0, torch.ones_like(s), s)
    q = (b / s[..., None]).to(torch.float8_e4m3fn)
    return (q.to(torch.float64) * s[..., None].to(torch.float64)).reshape(v32.shape)


def dense_ffn(ex, x_bf16: torch.Tensor):
    xh = torch_quant(x_bf16.to(torch.float32)).numpy()
    g = xh @ dense(ex.gate_codes, ex.gate_scales).T
    u = xh @ dense(ex.up_codes, ex.up_scales).T
    h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
    hh = torch_quant(torch.from_numpy(h)).numpy()
    return hh @ dense(ex.down_codes, ex.down_scales).T


def test_gemv_integer_exact_unit_scales():
    rng = np.random.default_rng(10)
    rows, K = 64, 512
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = np.full((rows, K // 32), 127, np.uint8)
    x = rng.integers(-448, 449, K).astype(np.int64)
    w2 = (2 * E2M1[_nibbles(codes)]).astype(np.int64)  # integers
    ref = (w2 @ x).astype(np.float64) / 2
    got = oracle.fp4_gemv(codes, scales, x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_gemv_integer_exact_block_scales():
    rng = np.random.default_rng(11)
    rows, K = 48, 1024
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = rng.integers(121, 125, (rows, K // 32), dtype=np.uint8)
    x = rng.integers(-448, 449, K).astype(np.int64)
    # 2 * e2m1 * 2^(b-127) * 2^7 = integer for b >= 121
    w_int = (2 * E2M1[_nibbles(codes)]).astype(np.int64) * \
        np.left_shift(1, scales.astype(np.int64) - 121).repeat(32, axis=1)
    ref = (w_int @ x).astype(np.float64) / 128.0
    got = oracle.fp4_gemv(codes, scales, x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_gemv_scale_index_is_per_32_along_reduction():
    # One scale byte changed at column block 3 of row 2 must change only row 2's output.
    rng = np.random.default_rng(12)
    codes = rng.integers(0, 256, (4, 128), dtype=np.uint8)
    scales = np.full((4, 8), 124, np.uint8)
    x = np.ones(256)
    base = oracle.fp4_gemv(codes, scales, x)
    scales[2, 3] = 125
    got = oracle.fp4_gemv(codes, scales, x)
    blk = E2M1[_nibbles(codes)[2, 96:128]].sum() * 2.0 ** (124 - 127)
    assert np.array_equal(got[[0, 1, 3]], base[[0, 1, 3]])
    assert abs(got[2] - (base[2] + blk)) < 1e-12


def _tiny_weights(E, d, f, seed=5):
    return {e: synth.host_expert(seed, 0, e, d, f) for e in range(E + 1)}


def test_expert_ffn_matches_dense_library_ffn():
    d, f = 256, 128
    ex = synth.host_expert(3, 0, 1, d, f)
    x = synth.gen_x(5, d, seed=9)
    qx, sx = oracle.act_quant(x)
    y = oracle.expert_ffn(ex, d, f, qx, sx)
    ref = dense_ffn(ex, x)
    assert np.allclose(y, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


def test_layer_k1_equals_dense_ffn_plus_shared():
    T, E, k, d, f = 6, 4, 1, 256, 128
    experts = _tiny_weights(E, d, f)
    x = synth.gen_x(T, d, seed=21)
    s = synth.gen_scores_uniform(T, E, seed=22)
    idx, w = oracle.route_topk(s.numpy(), k)
    assert (w == 1.0).all()
    y_pair, y_sh, out = oracle.moe_layer(x, E, k, d, f, experts, idx, w)
    for t in range(T):
        ref = dense_ffn(experts[E], x[t:t + 1]) + dense_ffn(experts[int(idx[t, 0])], x[t:t + 1])
        assert np.allclose(out[t], ref[0], rtol=1e-10, atol=1e-12 * np.abs(ref).max())


def test_layer_tiny_matches_dense_library_layer():
    w_ = synth.WORKLOADS["tiny"]
    experts = _tiny_weights(w_.E, w_.d, w_.f, seed=w_.seed())
    x, s = synth.gen_layer_inputs(w_)
    idx, w = oracle.route_topk(s.numpy(), w_.k)
    _, _, out = oracle.moe_layer(x, w_.E, w_.k, w_.d, w_.f, experts, idx, w)
    ref = np.zeros((w_.T, w_.d))
    for t in range(w_.T):
        acc = dense_ffn(experts[w_.E], x[t:t + 1])[0]
        for j in range(w_.k):
            acc = acc + w[t, j] * dense_ffn(experts[int(idx[t, j])], x[t:t + 1])[0]
        ref[t] = acc
    assert np.allclose(out, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


def test_layer_token_permutation_invariance():
    T, E, k, d, f = 9, 8, 3, 256, 128
    experts = _tiny_weights(E, d, f, seed=33)
    x = synth.gen_x(T, d, seed=34)
    s = synth.gen_scores_zipf(T, E, 1.0, seed=35)
    idx, w = oracle.route_topk(s.numpy(), k)
    yp, ysh, out = oracle.moe_layer(x, E, k, d, f, experts, idx, w)
    p = np.random.default_rng(36).permutation(T)
    idx2, w2 = oracle.route_topk(s.numpy()[p], k)
    assert np.array_equal(idx2, idx[p])
    yp2, ysh2, out2 = oracle.moe_layer(x[torch.from_numpy(p)], E, k, d, f, experts, idx2, w2)
    assert np.array_equal(out2, out[p]) and np.array_equal(ysh2, ysh[p])
    assert np.array_equal(yp2.reshape(T, k, d), yp.reshape(T, k, d)[p])


def test_moe_tokens_agrees_with_moe_layer():
    T, E, k, d, f = 7, 8, 2, 256, 128
    experts = _tiny_weights(E, d, f, seed=41)
    x = synth.gen_x(T, d, seed=42)
    s = synth.gen_scores_uniform(T, E, seed=43)
    idx, w = oracle.route_topk(s.numpy(), k)
    yp, ysh, out = oracle.moe_layer(x, E, k, d, f, experts, idx, w)
    sel = [0, 3, 6]
    yp2, ysh2, out2 = oracle.moe_tokens(x, E, k, d, f, experts, idx, w, sel)
    assert np.array_equal(out2, out[sel]) and np.array_equal(ysh2, ysh[sel])
    assert np.array_equal(yp2, yp.reshape(T, k, d)[sel])


def test_combine_weights_sum_to_one_makes_constant_experts_pass_through():
    # if every routed expert returns the same vector v, out = y_sh + v (Σw = 1)
    T, k, d = 3, 6, 16
    rng = np.random.default_rng(50)
    v = rng.normal(size=d)
    ysh = rng.normal(size=(T, d))
    s = synth.gen_scores_uniform(T, 256, seed=51)
    _, w = oracle.route_topk(s.numpy(), k)
    out = oracle.combine(ysh, np.broadcast_to(v, (T, k, d)).copy(), w)
    assert np.allclose(out, ysh + v, rtol=1e-14, atol=1e-14)
