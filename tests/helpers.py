"""Shared helpers for the parity tests: seeded inputs for both sides, oracle references,
and the comparison rules (bit-exact for integers and codes; rel-L2 <= 1e-3 and
max-abs <= 1e-2 * max|ref| for the floating-point layer outputs)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

REL_L2 = 1e-3
MAX_ABS_FRAC = 1e-2


def close_report(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / (nref if nref > 0 else 1.0)
    mabs = float(np.abs(err).max()) if err.size else 0.0
    bound = MAX_ABS_FRAC * (float(np.abs(ref).max()) if ref.size else 0.0)
    return rel, mabs, bound


def assert_close(got, ref, what=""):
    rel, mabs, bound = close_report(got, ref)
    assert np.isfinite(np.asarray(got, np.float64)).all(), f"{what}: non-finite output"
    assert rel <= REL_L2 and mabs <= bound, \
        f"{what}: rel-L2 {rel:.3e} (<= {REL_L2}), max-abs {mabs:.3e} (<= {bound:.3e})"


def device_weights(seed, layer, E, d, f):
    import bit_moe_routed_b200 as bm
    return bm.LayerWeights.from_dict(synth.device_layer_weights(seed, layer, E, d, f))


def host_experts(seed, layer, d, f, experts):
    return {int(e): synth.host_expert(seed, layer, int(e), d, f) for e in experts}


def oracle_layer_tokens(x, scores, k, E, d, f, seed, layer, tokens):
    """Oracle routing + outputs for selected tokens; weights regenerated on the host."""
    idx, w = oracle.route_topk(scores.numpy(), k)
    need = set(idx[tokens].ravel().tolist()) | {E}
    ex = host_experts(seed, layer, d, f, need)
    y_pair, y_sh, out = oracle.moe_tokens(x, E, k, d, f, ex, idx, w, tokens)
    return idx, w, y_pair, y_sh, out


def gpu_layer(x, scores, k, weights, ws=None):
    import bit_moe_routed_b200 as bm
    r = bm.forward(x.cuda(), scores.cuda(), k, weights, ws)
    bm.sync_status()
    return {kk: v.cpu() for kk, v in r.items()}


def check_layer(g, x, scores, k, E, d, f, seed, layer, tokens, label=""):
    """Compare GPU layer results against the oracle on the given tokens."""
    idx, w, y_pair, y_sh, out = oracle_layer_tokens(x, scores, k, E, d, f, seed, layer, tokens)
    assert np.array_equal(g["idx"].numpy(), idx), f"{label}: routing indices differ"
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    assert np.array_equal(g["counts"].numpy(), counts), f"{label}: counts"
    assert np.array_equal(g["offsets"].numpy(), offsets), f"{label}: offsets"
    assert np.array_equal(g["perm"].numpy(), perm), f"{label}: perm"
    assert np.array_equal(g["pos"].numpy(), pos), f"{label}: pos"
    assert np.allclose(g["w"].numpy(), w, rtol=2e-6, atol=1e-7), f"{label}: gate weights"
    tok = np.asarray(tokens)
    y_gpu = g["y"].numpy()[pos.reshape(-1, k)[tok]]  # [n, k, d]
    assert_close(y_gpu, y_pair, f"{label}: y_routed")
    assert_close(g["y_shared"].numpy()[tok], y_sh, f"{label}: y_shared")
    assert_close(g["out"].numpy()[tok], out, f"{label}: out")
