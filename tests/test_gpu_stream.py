"""GPU checks of expert streaming (moe_forward_streamed): routed experts in pinned host
memory, an HBM cache of S slots.  Over a sequence of tokens the results must equal
moe_forward's on the resident layer bit for bit (the same kernel on the same bytes), and
after every step the cache's tables (expert -> slot, slot -> expert, last use) and its hit
and miss counts must equal the oracle's LRU model (oracle.lru_cache_steps) on the same
selections."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import device_weights

pytestmark = pytest.mark.gpu
bm = pytest.importorskip("bit_moe_routed_b200")


def run_sequence(E, k, d, f, S, n_tok, seed, zipf_s=1.2):
    W = device_weights(seed, 0, E, d, f)
    host = bm.HostExperts.from_layer(W)
    cache = bm.ExpertCache(E, S, d, f, W)
    ws = bm.alloc_workspace(1, k, E, d, f)
    ws2 = bm.alloc_workspace(1, k, E, d, f)
    sels = []
    for n in range(n_tok):
        x = synth.gen_x(1, d, seed=seed * 100 + n)
        s = synth.gen_scores_zipf(1, E, zipf_s, seed=seed * 100 + n)
        a = bm.forward_streamed(x.cuda(), s.cuda(), k, host, cache, ws)
        a = {kk: v.clone() for kk, v in a.items()}
        b = bm.forward(x.cuda(), s.cuda(), k, W, ws2)
        bm.sync_status()
        for name in ("idx", "w", "counts", "offsets", "perm", "pos", "y", "y_shared", "out"):
            assert torch.equal(a[name].cpu(), b[name].cpu()[:a[name].shape[0]]), f"token {n}: {name}"
        idx, _ = oracle.route_topk(s.numpy(), k)
        sels.append(idx[0].tolist())
        out, (slot_of, expert_of, last_use) = oracle.lru_cache_steps(sels, E, S)
        assert cache.slot_of.cpu().tolist() == slot_of, f"token {n}: slot_of"
        assert cache.expert_of.cpu().tolist() == expert_of, f"token {n}: expert_of"
        assert cache.last_use.cpu().tolist() == last_use, f"token {n}: last_use"
    hits = sum(len(h) for h, _, _ in out)
    misses = sum(len(m) for _, m, _ in out)
    assert cache.stats.cpu().tolist() == [hits, misses]
    return hits, misses


def test_streamed_decode_equals_resident_and_follows_lru():
    hits, misses = run_sequence(E=128, k=6, d=4096, f=2048, S=24, n_tok=24, seed=5)
    print(f"STREAM E=128 k=6 S=24: {hits} hits, {misses} misses over 24 tokens")
    assert hits > 0 and misses > 0


@pytest.mark.parametrize("E,k,d,f,S", [(32, 2, 2048, 1024, 4), (16, 4, 1024, 512, 4)])
def test_streamed_small_caches(E, k, d, f, S):
    run_sequence(E, k, d, f, S, n_tok=16, seed=E + S)


def test_cache_with_fewer_slots_than_k_is_rejected():
    E, k, d, f, S = 16, 4, 1024, 512, 3
    W = device_weights(2, 0, E, d, f)
    host = bm.HostExperts.from_layer(W)
    cache = bm.ExpertCache(E, S, d, f, W)
    x = synth.gen_x(1, d, seed=1).cuda()
    s = synth.gen_scores_uniform(1, E, seed=1).cuda()
    with pytest.raises(bm.MoeError) as ei:
        bm.forward_streamed(x, s, k, host, cache)
    assert ei.value.code == bm.MOE_ERR_INVALID_ARG


def test_pageable_host_arrays_are_rejected():
    """The copy kernel reads host memory directly: pageable arrays must be refused on the
    host (no kernel runs)."""
    E, k, d, f, S = 16, 2, 1024, 512, 4
    W = device_weights(4, 0, E, d, f)
    host = bm.HostExperts.from_layer(W)
    host.gate_codes = host.gate_codes.clone()  # a pageable copy
    assert not host.gate_codes.is_pinned()
    cache = bm.ExpertCache(E, S, d, f, W)
    x = synth.gen_x(1, d, seed=1).cuda()
    s = synth.gen_scores_uniform(1, E, seed=1).cuda()
    with pytest.raises(bm.MoeError) as ei:
        bm.forward_streamed(x, s, k, host, cache)
    assert ei.value.code == bm.MOE_ERR_INVALID_ARG
