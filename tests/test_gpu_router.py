"""Router scoring + top-k (moe_router_topk) against the oracle.

The scores are fp32 sums of exact bf16 x bf16 products, summed per 128-element chunk and
then in a fixed chunk and warp order, so each one is within D * 2^-23 * sum_i |x_i w_i|
of the oracle's double sum, D = 128 + d/128 + 8 (the same derivation as the FFN's bound).
The selection is then exact on the GPU's own scores (bit-exact against the oracle's top-k
of those scores) and equals the oracle's selection on its own scores except where the k-th
and (k+1)-th scores lie within twice that bound (both selections are then correct)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import U23, acc_depth, assert_within

pytestmark = pytest.mark.gpu

bm = pytest.importorskip("bit_moe_routed_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    bm.lib()


def _check(x, wr, k, tokens):
    T, d = x.shape
    E = wr.shape[0]
    scores, idx, w = bm.router_topk(x.cuda(), wr.cuda(), k)
    bm.sync_status()
    sg = scores.cpu().numpy()
    tok = np.asarray(tokens)
    so = oracle.router_scores(x[tok], wr)
    absx = x[tok].float().abs().to(torch.bfloat16)
    absw = wr.float().abs().to(torch.bfloat16)
    bound = 1.01 * acc_depth(d) * U23 * oracle.router_scores(absx, absw)
    worst = assert_within(sg[tok], so, bound, "router scores")
    # the selection on the GPU's own scores: bit-exact
    io, wo = oracle.route_topk(sg[tok], k)
    assert np.array_equal(idx.cpu().numpy()[tok], io), "top-k of the GPU's scores"
    assert np.allclose(w.cpu().numpy()[tok], wo, rtol=2e-6, atol=1e-7), "gate weights"
    # against the oracle's own selection: equal, or a near-tie at the k-th place
    ref, _ = oracle.route_topk(so.astype(np.float32), k)
    ties = 0
    for i in range(len(tok)):
        if set(io[i]) == set(ref[i]):
            continue
        order = np.sort(so[i])[::-1]
        gap = order[k - 1] - order[k]
        assert gap <= 2 * bound[i].max(), f"token {tok[i]}: selection differs, gap {gap:.3e}"
        kth = order[k]
        for e in io[i]:
            assert so[i, e] >= kth - 2 * bound[i, e], f"token {tok[i]}: expert {e} not in a top-{k}"
        ties += 1
    print(f"ROUTER T={T} E={E} d={d} k={k}: {len(tok)} tokens, worst err/bound {worst:.2e}, "
          f"near-tie selections {ties}")


@pytest.mark.parametrize("T,E,d,k", [(1, 256, 4096, 6), (7, 64, 512, 4), (64, 256, 4096, 6),
                                     (33, 1024, 1024, 8), (5, 3, 128, 2)])
def test_router_topk_against_oracle(T, E, d, k):
    x = synth.gen_x(T, d, seed=T + E + d)
    wr = synth.gen_router_weights(E, d, seed=T + E)
    _check(x, wr, k, list(range(T)))


def test_router_topk_prefill_sampled():
    T, E, d, k = 4096, 256, 4096, 6
    x = synth.gen_x(T, d, seed=4242)
    wr = synth.gen_router_weights(E, d, seed=4243)
    rng = np.random.default_rng(1)
    tokens = sorted(set([0, 15, 16, T - 1] + rng.integers(0, T, 60).tolist()))
    _check(x, wr, k, tokens)
