"""Pins for the oracle's routing (top-k) and dispatch (stable grouping), CPU only.

Checked against torch.topk / stable torch.sort / bincount (library routines),
a closed-form gating example, and the invariants of a permutation.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


@pytest.mark.parametrize("T,E,k", [(1, 256, 6), (4, 8, 2), (64, 256, 6), (33, 17, 5), (5, 3, 3)])
def test_topk_matches_torch_topk(T, E, k):
    s = synth.gen_scores_uniform(T, E, seed=T * 31 + E)
    idx, w = oracle.route_topk(s.numpy(), k)
    tv, ti = torch.topk(s, k, dim=1, largest=True, sorted=True)
    assert np.array_equal(idx, ti.numpy().astype(np.int32))
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert (np.diff(w, axis=1) <= 0).all()


def test_topk_zipf_scores_match_torch_topk():
    s = synth.gen_scores_zipf(64, 256, 1.0, seed=7)
    idx, _ = oracle.route_topk(s.numpy(), 6)
    assert np.array_equal(idx, torch.topk(s, 6, dim=1).indices.numpy().astype(np.int32))


def test_topk_ties_go_to_lower_index():
    s = np.array([[0.5, 0.9, 0.9, 0.1, 0.9]], np.float32)
    idx, _ = oracle.route_topk(s, 4)
    assert idx.tolist() == [[1, 2, 4, 0]]


def test_gate_weights_closed_form():
    # sigmoid(ln 3) = 3/4, sigmoid(0) = 1/2 -> renormalised 0.6 / 0.4
    s = np.array([[0.0, math.log(3.0), -5.0]], np.float32)
    idx, w = oracle.route_topk(s, 2)
    assert idx.tolist() == [[1, 0]]
    ln3 = float(np.float32(math.log(3.0)))
    p = 1 / (1 + math.exp(-ln3))
    assert abs(w[0, 0] - p / (p + 0.5)) < 1e-15 and abs(w[0, 0] - 0.6) < 1e-7
    # k = 1 gives weight exactly 1
    _, w1 = oracle.route_topk(s, 1)
    assert w1[0, 0] == 1.0


@pytest.mark.parametrize("T,E,k", [(1, 256, 6), (4, 8, 2), (4096, 256, 6), (7, 5, 5)])
def test_dispatch_matches_stable_sort(T, E, k):
    s = synth.gen_scores_zipf(T, E, 1.2, seed=T + E)
    idx, _ = oracle.route_topk(s.numpy(), k)
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    flat = torch.from_numpy(idx.reshape(-1).astype(np.int64))
    ref_perm = torch.sort(flat, stable=True).indices.numpy()
    assert np.array_equal(perm, ref_perm)
    assert np.array_equal(counts, torch.bincount(flat, minlength=E).numpy())
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(pos[perm], np.arange(T * k))
    keys = idx.reshape(-1)[perm]
    assert (np.diff(keys) >= 0).all()


def test_dispatch_empty_and_single_expert():
    idx = np.zeros((5, 1), np.int32)  # every token on expert 0
    counts, offsets, perm, pos = oracle.dispatch(idx, 4)
    assert counts.tolist() == [5, 0, 0, 0] and offsets.tolist() == [0, 5, 5, 5, 5]
    assert perm.tolist() == [0, 1, 2, 3, 4]
    counts, offsets, perm, pos = oracle.dispatch(np.zeros((0, 3), np.int32), 4)
    assert counts.tolist() == [0, 0, 0, 0] and offsets.tolist() == [0] * 5 and perm.size == 0


# ---------------------------------------------------------------- router scores (NEXT-1)
def _bf16(a):
    return torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_router_scores_match_float64_matmul():
    """Against numpy's float64 matmul of the bf16-decoded inputs (a library routine)."""
    rng = np.random.default_rng(5)
    x = _bf16(rng.normal(size=(7, 384)))
    w = _bf16(rng.normal(size=(40, 384)) * 0.05)
    got = oracle.router_scores(x, w)
    ref = x.float().numpy().astype(np.float64) @ w.float().numpy().astype(np.float64).T
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_router_scores_closed_forms():
    """One-hot tokens pick out columns of W; integer inputs give exact integer scores."""
    d, E = 64, 9
    rng = np.random.default_rng(6)
    w = _bf16(rng.integers(-8, 9, size=(E, d)))
    x = np.zeros((3, d), np.float32)
    x[0, 5] = 1.0
    x[1, 63] = -2.0
    x[2] = rng.integers(-4, 5, size=d)
    s = oracle.router_scores(_bf16(x), w)
    wf = w.float().numpy().astype(np.float64)
    assert np.array_equal(s[0], wf[:, 5])
    assert np.array_equal(s[1], -2.0 * wf[:, 63])
    assert np.array_equal(s[2], np.array([int(np.dot(x[2].astype(np.int64),
                                                      wf[e].astype(np.int64))) for e in range(E)],
                                         dtype=np.float64))


def test_router_then_topk_selects_the_largest_dot_products():
    """A planted winner: the experts whose rows align with the token are chosen in order."""
    d, E, k = 128, 16, 3
    rng = np.random.default_rng(7)
    x = rng.normal(size=(1, d)).astype(np.float32)
    w = rng.normal(size=(E, d)).astype(np.float32) * 0.01
    w[11] = x[0]
    w[2] = 0.5 * x[0]
    w[7] = 0.25 * x[0]
    s = oracle.router_scores(_bf16(x), _bf16(w)).astype(np.float32)
    idx, _ = oracle.route_topk(s, k)
    assert idx.tolist() == [[11, 2, 7]]
