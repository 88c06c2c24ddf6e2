"""GPU parity of the single-token layer with 2-bit routed experts (moe_forward_q2) against
the oracle: routing, dispatch and the token's codes bit for bit; the re-quantised h of
every (token, expert) vector against the oracle's codes under the derived tie rule; the
fp32 h, y and out within their a-priori bounds (the oracle decodes the 2-bit codes,
tests/test_oracle_q2.py pins it)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import check_layer, device_weights, gpu_layer_q2, host_experts, host_experts_q2

pytestmark = pytest.mark.gpu
bm = pytest.importorskip("bit_moe_routed_b200")


def q2_device(seed, layer, E, d, f):
    return bm.Q2Experts.from_dict(synth.device_layer_weights_q2(seed, layer, E, d, f))


def run_q2(E, k, d, f, seed, label, x=None, scores=None):
    if x is None:
        x = synth.gen_x(1, d, seed=seed + 1)
    if scores is None:
        scores = synth.gen_scores_uniform(1, E, seed=seed + 2)
    W = device_weights(seed, 0, E, d, f)
    Q = q2_device(seed, 0, E, d, f)
    g = gpu_layer_q2(x, scores, k, W, Q)
    idx, _ = oracle.route_topk(scores.numpy(), k)
    experts = host_experts_q2(seed, 0, d, f, set(idx.ravel().tolist()))
    experts.update(host_experts(seed, 0, d, f, [E]))  # the shared expert stays FP4
    return check_layer(g, x, scores, k, E, d, f, seed, 0, [0], label=label, experts=experts)


def test_q2_decode_layer_matches_oracle():
    w = synth.WORKLOADS["decode_t1"]
    x, s = synth.gen_layer_inputs(w, 0)
    run_q2(w.E, w.k, w.d, w.f, w.seed(0), "decode_t1_q2", x=x, scores=s)


@pytest.mark.parametrize("E,k,d,f", [(8, 2, 2048, 2048), (16, 1, 2048, 2048),
                                     (64, 7, 2048, 2048), (512, 3, 4096, 2048)])
def test_q2_shapes(E, k, d, f):
    run_q2(E, k, d, f, seed=E + k + d // 512 + f // 256, label=f"q2 E={E} k={k} d={d} f={f}")


def test_q2_rejects_shapes_it_cannot_run():
    E, k, d, f = 8, 2, 1024, 2048  # d not a multiple of 2048
    W = device_weights(3, 0, E, d, f)
    Q = q2_device(3, 0, E, d, f)
    x = synth.gen_x(1, d, seed=4).cuda()
    s = synth.gen_scores_uniform(1, E, seed=5).cuda()
    with pytest.raises(bm.MoeError) as ei:
        bm.forward_q2(x, s, k, W, Q)
    assert ei.value.code == bm.MOE_ERR_INVALID_ARG


def test_q2_repeated_launches_agree():
    """Two launches with the same inputs give the same bits (no timing dependence)."""
    E, k, d, f = 64, 4, 2048, 2048
    W = device_weights(9, 0, E, d, f)
    Q = q2_device(9, 0, E, d, f)
    x = synth.gen_x(1, d, seed=10).cuda()
    s = synth.gen_scores_uniform(1, E, seed=11).cuda()
    a = bm.forward_q2(x, s, k, W, Q)
    a = {kk: v.clone() for kk, v in a.items()}
    b = bm.forward_q2(x, s, k, W, Q)
    bm.sync_status()
    for name in ("idx", "w", "y", "y_shared", "out"):
        assert torch.equal(a[name], b[name]), name
