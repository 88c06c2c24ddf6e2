"""GPU parity: the CUDA library (through the C ABI) against the oracle.

Routing indices, the dispatch permutation, offsets and the quantised activation codes
and scales must match bit-exactly; the re-quantised hidden state must match the oracle's
codes up to counted ties, and FFN outputs (y_routed, y_shared, out) must lie within
derived element-wise bounds of the oracle evaluated on the GPU's codes and within rel-L2
<= 1e-3, max-abs <= 1e-2 * max|ref| (helpers.py states the rules).  Small shapes are
compared in full; decode_t64 on all its tokens; prefill on 64 tokens chosen to cover the
tile kernels' edges (the hottest expert's last tile, the stream-K tail, the last rows of
tiles), which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import (assert_close, check_layer, device_weights, gpu_layer, host_experts,
                     tile_sample_tokens)

pytestmark = pytest.mark.gpu

bm = pytest.importorskip("bit_moe_routed_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    bm.lib()
    yield
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- routing and dispatch
@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_route_and_dispatch_bit_exact(name):
    w_ = synth.WORKLOADS[name]
    s = synth.gen_scores(w_, 0)
    idx_o, w_o = oracle.route_topk(s.numpy(), w_.k)
    idx, w = bm.route_topk(s.cuda(), w_.k)
    counts, offsets, perm, pos = bm.dispatch(idx, w_.E)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.allclose(w.cpu().numpy(), w_o, rtol=2e-6, atol=1e-7)
    c_o, off_o, perm_o, pos_o = oracle.dispatch(idx_o, w_.E)
    assert np.array_equal(counts.cpu().numpy(), c_o)
    assert np.array_equal(offsets.cpu().numpy(), off_o)
    assert np.array_equal(perm.cpu().numpy(), perm_o)
    assert np.array_equal(pos.cpu().numpy(), pos_o)


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (5, 3, 3), (37, 1024, 8), (300, 512, 32),
                                   (2000, 64, 6)])
def test_route_and_dispatch_odd_shapes(T, E, k):
    s = synth.gen_scores_uniform(T, E, seed=T + E + k)
    idx_o, _ = oracle.route_topk(s.numpy(), k)
    idx, _ = bm.route_topk(s.cuda(), k)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    counts, offsets, perm, pos = bm.dispatch(idx, E)
    c_o, off_o, perm_o, pos_o = oracle.dispatch(idx_o, E)
    assert np.array_equal(offsets.cpu().numpy(), off_o)
    assert np.array_equal(perm.cpu().numpy(), perm_o)


@pytest.mark.parametrize("T,E,k", [(1366, 256, 6), (4096, 256, 6), (2000, 1024, 8),
                                   (9000, 7, 1), (4096, 256, 6)])
def test_multi_cta_dispatch_matches_oracle_and_one_cta(T, E, k):
    """Large batches: the multi-CTA dispatch (per-segment counts, then a scatter) gives the
    oracle's stable permutation, bit for bit, and the same as the one-CTA kernel."""
    assert bm.lib().moe_dispatch_workspace_size(T, k, E) > 0
    s = synth.gen_scores_zipf(T, E, 1.2, seed=T + E) if E > 8 else \
        synth.gen_scores_uniform(T, E, seed=T)
    idx_o, _ = oracle.route_topk(s.numpy(), k)
    idx = torch.from_numpy(idx_o).cuda()
    multi = bm.dispatch(idx, E)
    one = bm.dispatch(idx, E, multi=False)
    ref = oracle.dispatch(idx_o, E)
    for a, b_, r, name in zip(multi, one, ref, ("counts", "offsets", "perm", "pos")):
        assert np.array_equal(a.cpu().numpy(), r), f"multi-CTA {name}"
        assert torch.equal(a, b_), f"multi vs one CTA: {name}"


def test_route_ties_go_to_lower_index():
    s = torch.tensor([[0.5, 0.9, 0.9, 0.1, 0.9] + [0.0] * 27], dtype=torch.float32)
    idx, _ = bm.route_topk(s.cuda(), 4)
    assert idx.cpu().tolist() == [[1, 2, 4, 0]]


def test_dispatch_one_expert_and_empty():
    idx = torch.zeros((300, 1), dtype=torch.int32, device="cuda")
    counts, offsets, perm, pos = bm.dispatch(idx, 4)
    assert counts.cpu().tolist() == [300, 0, 0, 0]
    assert offsets.cpu().tolist() == [0, 300, 300, 300, 300]
    assert perm.cpu().tolist() == list(range(300))
    counts, offsets, _, _ = bm.dispatch(torch.zeros((0, 2), dtype=torch.int32, device="cuda"), 4)
    assert counts.cpu().tolist() == [0] * 4 and offsets.cpu().tolist() == [0] * 5


# ---------------------------------------------------------------- activation quantisation
@pytest.mark.parametrize("T,d", [(1, 128), (3, 256), (64, 4096), (17, 8192), (4096, 4096)])
def test_act_quant_bit_exact(T, d):
    x = synth.gen_x(T, d, seed=T * 7 + d)
    q_o, s_o = oracle.act_quant(x)
    q, s = bm.act_quant(x.cuda())
    assert np.array_equal(s.cpu().numpy(), s_o)
    assert np.array_equal(q.cpu().numpy(), q_o)


def test_act_quant_special_rows():
    d = 512
    rows = [torch.zeros(d), torch.full((d,), 448.0), torch.full((d,), -1e30),
            torch.tensor([1e-30, -1e-30] * (d // 2)), torch.linspace(-3, 3, d)]
    x = torch.stack(rows)
    x[3, 0] = 1.0  # tiny values next to a large one round to +-0
    x = x.to(torch.bfloat16)
    q_o, s_o = oracle.act_quant(x)
    q, s = bm.act_quant(x.cuda())
    assert np.array_equal(s.cpu().numpy(), s_o)
    assert np.array_equal(q.cpu().numpy(), q_o)


def test_prepare_rows_for_any_permutation():
    """The prepare step from 2048 pairs (the tile path's per-token form: the inverse of the
    permutation, then each token quantised once) on a shuffled permutation, not the
    dispatch's: row r holds token perm[r] // k's codes and scales, rows P.. the tokens in
    order, bit for bit.  Then a permutation with an entry out of range is flagged."""
    T, E, k, d, f = 512, 64, 6, 1024, 512
    P = T * k
    x = synth.gen_x(T, d, seed=515)
    s = synth.gen_scores_uniform(T, E, 516)
    W = device_weights(517, 0, E, d, f)
    assert bm.ffn_path(T, k, W) == bm.PATH_TILES
    idx, _ = bm.route_topk(s.cuda(), k)
    _, offsets, _, _ = bm.dispatch(idx, E)
    perm = torch.from_numpy(np.random.default_rng(518).permutation(P).astype(np.int32))
    ws = bm.alloc_workspace(T, k, E, d, f)
    bm.ffn_prepare(x.cuda(), k, W, offsets, perm.cuda(), ws)
    bm.sync_status()
    v = bm.workspace_views(ws, T, k, E, d, f)
    q_o, s_o = oracle.act_quant(x)
    src = np.concatenate([perm.numpy() // k, np.arange(T)])
    assert np.array_equal(v["qx"].cpu().numpy(), q_o[src])
    assert np.array_equal(v["sx"].cpu().numpy(), s_o[src])
    bad = perm.clone()
    bad[7] = P + 3
    bm.ffn_prepare(x.cuda(), k, W, offsets, bad.cuda(), ws)
    with pytest.raises(bm.MoeError):
        bm.sync_status()
    bm.sync_status()  # the status word is cleared once reported


# ---------------------------------------------------------------- whole layer, small shapes
def _small_layer(T, E, k, d, f, routing="uniform", seed=5, zero_rows=(), calls=False):
    x = synth.gen_x(T, d, seed=seed)
    for r in zero_rows:
        x[r] = 0
    s = synth.gen_scores_uniform(T, E, seed + 1) if routing == "uniform" else \
        synth.gen_scores_zipf(T, E, 1.2, seed + 1)
    W = device_weights(seed, 0, E, d, f)
    g = gpu_layer(x, s, k, W, calls=calls)
    check_layer(g, x, s, k, E, d, f, seed, 0, list(range(T)),
                f"T={T} E={E} k={k} d={d} f={f}" + (" (four calls)" if calls else ""))


def test_layer_tiny_workload():
    w_ = synth.WORKLOADS["tiny"]
    x, s = synth.gen_layer_inputs(w_)
    W = device_weights(w_.seed(), 0, w_.E, w_.d, w_.f)
    g = gpu_layer(x, s, w_.k, W)
    check_layer(g, x, s, w_.k, w_.E, w_.d, w_.f, w_.seed(), 0, list(range(w_.T)), "tiny")


@pytest.mark.parametrize("T,E,k,d,f,routing", [
    (1, 4, 1, 128, 128, "uniform"),
    (3, 8, 2, 256, 128, "uniform"),
    (33, 16, 4, 512, 256, "zipf"),      # crosses the small/large tile switch
    (130, 8, 3, 256, 384, "zipf"),      # groups larger than one 112-row tile
    (250, 32, 6, 384, 256, "uniform"),
])
def test_layer_ragged_shapes(T, E, k, d, f, routing):
    _small_layer(T, E, k, d, f, routing, seed=T + E)


@pytest.mark.parametrize("T,E,k,d,f,routing", [
    (2, 8, 2, 512, 512, "uniform"),
    (7, 16, 3, 1024, 512, "zipf"),       # one slot per expert, fewer than 8 tokens
    (16, 32, 4, 512, 1024, "zipf"),      # the shared expert in two slots
    (33, 16, 6, 1024, 512, "zipf"),      # hot experts in several slots
    (64, 256, 6, 2048, 1024, "zipf"),    # CTA ranges over many slots
])
def test_batched_gemv_shapes(T, E, k, d, f, routing):
    """2 <= T <= 64 with d, f multiples of 512: the batched FP4 GEMV kernels."""
    _small_layer(T, E, k, d, f, routing, seed=T + E + d)


def test_batched_gemv_all_tokens_one_expert():
    """40 tokens on one routed expert: five slots of 8 rows re-read its weights."""
    T, E, k, d, f = 40, 8, 1, 512, 512
    x = synth.gen_x(T, d, seed=95)
    s = synth.gen_scores_uniform(T, E, seed=96)
    s[:, 5] += 10.0
    W = device_weights(97, 0, E, d, f)
    g = gpu_layer(x, s, k, W)
    assert g["counts"].tolist()[5] == T
    check_layer(g, x, s, k, E, d, f, 97, 0, list(range(T)), "one expert, batched GEMV")


def test_layer_zero_activations():
    _small_layer(6, 8, 2, 256, 128, seed=77, zero_rows=(0, 3))


def test_layer_all_tokens_one_expert():
    T, E, k, d, f = 240, 8, 1, 256, 256
    x = synth.gen_x(T, d, seed=90)
    s = synth.gen_scores_uniform(T, E, seed=91)
    s[:, 3] += 10.0  # every token picks expert 3: three token tiles of one expert
    W = device_weights(92, 0, E, d, f)
    g = gpu_layer(x, s, k, W)
    assert g["counts"].tolist()[3] == T
    check_layer(g, x, s, k, E, d, f, 92, 0, list(range(0, T, 7)), "one expert")


def test_layer_extreme_weights():
    """All codes +-6 with the largest scale used (2^-3), all codes 0, and mixed."""
    T, E, k, d, f = 5, 4, 2, 256, 128
    rng = np.random.default_rng(3)

    def mk(which):
        r, K = synth.matrix_shape(which, d, f)
        codes = np.full((E + 1, r, K // 2), 0x77, np.uint8)  # +6, +6
        codes[1] = 0xFF                                       # -6, -6
        codes[2] = 0x00                                       # zeros
        codes[3] = rng.integers(0, 256, codes[3].shape, dtype=np.uint8)
        scales = np.full((E + 1, r, K // 32), 124, np.uint8)
        scales[3] = rng.integers(121, 125, scales[3].shape, dtype=np.uint8)
        return codes, scales

    arrs = {}
    for name, which in (("gate", synth.GATE), ("up", synth.UP), ("down", synth.DOWN)):
        c, s_ = mk(which)
        arrs[f"{name}_codes"], arrs[f"{name}_scales"] = c, s_
    W = bm.LayerWeights.from_dict({kk: torch.from_numpy(v).cuda() for kk, v in arrs.items()})
    x = synth.gen_x(T, d, seed=11)
    s = synth.gen_scores_uniform(T, E, seed=12)
    g = gpu_layer(x, s, k, W)
    idx, w = oracle.route_topk(s.numpy(), k)
    ex = {e: synth.HostExpert(*(arrs[n][e] for n in (
        "gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales")))
        for e in range(E + 1)}
    y_pair, y_sh, out = oracle.moe_layer(x, E, k, d, f, ex, idx, w)
    assert np.array_equal(g["idx"].numpy(), idx)
    assert_close(g["out"].numpy(), out, "extreme weights: out")
    assert_close(g["y_shared"].numpy(), y_sh, "extreme weights: y_shared")


# ---------------------------------------------------------------- single-token GEMV path
@pytest.mark.parametrize("calls", [False, True], ids=["forward", "calls"])
@pytest.mark.parametrize("E,k,d,f", [
    (8, 2, 512, 512),       # one stage per row along d and along f
    (16, 4, 1024, 512),
    (32, 6, 512, 1536),     # three stages per down row
    (256, 6, 2048, 1024),   # CTA ranges that span two experts
    (1024, 8, 1024, 512),   # many experts: top-k over 32 scores per lane
    (64, 32, 512, 512),     # the most experts per token
])
def test_gemv_single_token_shapes(E, k, d, f, calls):
    _small_layer(1, E, k, d, f, "uniform", seed=E + d + f + k, calls=calls)


def test_single_token_paths_agree_bit_for_bit():
    """One token through moe_forward (one kernel, its CUDA-core form), the four calls (the
    FFN as one kernel), and the three exposed FFN stages (two GEMV kernels): identical
    results.  (The tensor-core form of moe_forward sums in another order: its own tests
    are in test_gpu_decode_tc.py.)"""
    E, k, d, f = 256, 6, 4096, 2048
    x = synth.gen_x(1, d, seed=61)
    s = synth.gen_scores_uniform(1, E, seed=62)
    W = device_weights(63, 0, E, d, f)
    bm.set_decode_engine(0)  # the default
    a = gpu_layer(x, s, k, W)
    b = gpu_layer(x, s, k, W, calls=True)
    xd, sd = x.cuda(), s.cuda()
    idx, gw = bm.route_topk(sd, k)
    counts, offsets, perm, pos = bm.dispatch(idx, E)
    ws = bm.alloc_workspace(1, k, E, d, f)
    y = torch.empty((k, d), dtype=torch.float32, device="cuda")
    ysh = torch.empty((1, d), dtype=torch.float32, device="cuda")
    bm.ffn_prepare(xd, k, W, offsets, perm, ws)
    bm.ffn_gate_up(1, k, W, ws)
    bm.ffn_down(1, k, W, y, ysh, ws)
    out = bm.combine(y, ysh, gw, pos)
    c = dict(idx=idx, w=gw, counts=counts, offsets=offsets, perm=perm, pos=pos, y=y,
             y_shared=ysh, out=out)
    c.update(bm.workspace_views(ws, 1, k, E, d, f))
    bm.sync_status()
    for name in ("idx", "w", "counts", "offsets", "perm", "pos", "y", "y_shared", "out", "qh",
                 "sh", "h"):
        assert torch.equal(a[name].cpu(), b[name].cpu()), f"forward vs calls: {name}"
        assert torch.equal(a[name].cpu(), c[name].cpu()), f"forward vs stages: {name}"
    for name in ("qx", "sx"):  # the single-token path writes row 0, the token
        assert torch.equal(a[name].cpu()[0], b[name].cpu()[0]), f"forward vs calls: {name}"
        assert torch.equal(a[name].cpu()[0], c[name].cpu()[0]), f"forward vs stages: {name}"


def test_single_token_repeated_expert_in_dispatch():
    """moe_expert_ffn at one token with an expert listed twice in topk_idx (a caller's own
    routing): both of its rows get the expert's output."""
    E, k, d, f = 8, 3, 512, 512
    x = synth.gen_x(1, d, seed=71)
    W = device_weights(72, 0, E, d, f)
    idx = torch.tensor([[5, 2, 5]], dtype=torch.int32, device="cuda")
    counts, offsets, perm, pos = bm.dispatch(idx, E)
    y, ysh = bm.expert_ffn(x.cuda(), k, W, offsets, perm)
    bm.sync_status()
    qx, sx = oracle.act_quant(x)
    ex = host_experts(72, 0, d, f, [2, 5, E])
    y_cpu = y.cpu().numpy()
    for j, e in enumerate([5, 2, 5]):
        yo = oracle.expert_ffn(ex[e], d, f, qx, sx)[0]
        assert_close(y_cpu[int(pos[j])], yo, f"pair {j} (expert {e})")
    assert_close(ysh.cpu().numpy()[0], oracle.expert_ffn(ex[E], d, f, qx, sx)[0], "shared")


def _custom_layer_check(T, E, k, d, f, arrs, seed, label):
    W = bm.LayerWeights.from_dict({kk: torch.from_numpy(v).cuda() for kk, v in arrs.items()})
    x = synth.gen_x(T, d, seed=seed)
    s = synth.gen_scores_uniform(T, E, seed=seed + 1)
    g = gpu_layer(x, s, k, W)
    idx, w = oracle.route_topk(s.numpy(), k)
    ex = {e: synth.HostExpert(*(arrs[n][e] for n in (
        "gate_codes", "gate_scales", "up_codes", "up_scales", "down_codes", "down_scales")))
        for e in range(E + 1)}
    y_pair, y_sh, out = oracle.moe_layer(x, E, k, d, f, ex, idx, w)
    assert np.array_equal(g["idx"].numpy(), idx)
    assert_close(g["out"].numpy(), out, f"{label}: out")
    assert_close(g["y_shared"].numpy(), y_sh, f"{label}: y_shared")


@pytest.mark.parametrize("gemv", [1, 0], ids=["gemv", "tiles"])
def test_wide_scale_range_single_token(gemv):
    """Block scales spread over 2^-40 .. 2^9 for gate/up and 2^-30 .. 2^-1 for down: more
    than the f16 range inside one 512-element span, and rows of very different size."""
    E, k, d, f = 8, 3, 1024, 512
    rng = np.random.default_rng(21)
    arrs = {}
    for name, which, lo, hi in (("gate", synth.GATE, 87, 137), ("up", synth.UP, 87, 137),
                                ("down", synth.DOWN, 97, 127)):
        r, K = synth.matrix_shape(which, d, f)
        arrs[f"{name}_codes"] = rng.integers(0, 256, (E + 1, r, K // 2), dtype=np.uint8)
        arrs[f"{name}_scales"] = rng.integers(lo, hi, (E + 1, r, K // 32), dtype=np.uint8)
    bm.set_gemv_max_tokens(gemv)
    try:
        _custom_layer_check(1, E, k, d, f, arrs, 31, "wide scales")
    finally:
        bm.set_gemv_max_tokens(bm.GEMV_MAX_TOKENS)


def test_extreme_weights_single_token():
    """All codes +-6 at scale 2^-3, all zeros, and rows whose 16 scales are 0 (2^-127)."""
    E, k, d, f = 4, 2, 512, 512
    rng = np.random.default_rng(4)
    arrs = {}
    for name, which in (("gate", synth.GATE), ("up", synth.UP), ("down", synth.DOWN)):
        r, K = synth.matrix_shape(which, d, f)
        codes = np.full((E + 1, r, K // 2), 0x77, np.uint8)
        codes[1] = 0xFF
        codes[2] = 0x00
        codes[3] = rng.integers(0, 256, codes[3].shape, dtype=np.uint8)
        scales = np.full((E + 1, r, K // 32), 124, np.uint8)
        scales[3] = rng.integers(121, 125, scales[3].shape, dtype=np.uint8)
        scales[3, ::7] = 0
        arrs[f"{name}_codes"], arrs[f"{name}_scales"] = codes, scales
    _custom_layer_check(1, E, k, d, f, arrs, 41, "extreme weights, T=1")


def test_device_generator_matches_host_generator():
    seed, layer, E, d, f = 1234, 3, 8, 256, 128
    dev = synth.device_layer_weights(seed, layer, E, d, f)
    host = synth.host_layer_weights(seed, layer, E, d, f)
    for kk in host:
        assert np.array_equal(dev[kk].cpu().numpy(), host[kk]), kk


# ---------------------------------------------------------------- full-size workloads
def _full_workload(name, tokens=None, n_sample=64, calls=False):
    w_ = synth.WORKLOADS[name]
    x, s = synth.gen_layer_inputs(w_, 0)
    W = device_weights(w_.seed(), 0, w_.E, w_.d, w_.f)
    oracle.set_threads(max(8, (__import__("os").cpu_count() or 8)))
    g = gpu_layer(x, s, w_.k, W, calls=calls)
    del W
    torch.cuda.empty_cache()
    if tokens is None:
        idx, _ = oracle.route_topk(s.numpy(), w_.k)
        tokens = tile_sample_tokens(idx, w_.E, n_sample, seed=w_.seed())
    check_layer(g, x, s, w_.k, w_.E, w_.d, w_.f, w_.seed(), 0, tokens, name)
    return g


@pytest.mark.parametrize("path", ["forward", "calls", "tiles"])
def test_decode_t1_full(path):
    """decode_t1 through moe_forward (one kernel), the four calls, and the tile kernels."""
    bm.set_gemv_max_tokens(0 if path == "tiles" else 1)
    try:
        _full_workload("decode_t1", [0], calls=path == "calls")
    finally:
        bm.set_gemv_max_tokens(bm.GEMV_MAX_TOKENS)


@pytest.mark.parametrize("path", ["gemv", "tiles"])
def test_decode_t64_zipf_all_tokens(path):
    """decode_t64 through the batched GEMV kernels and through the tile kernels."""
    bm.set_gemv_max_tokens(0 if path == "tiles" else bm.GEMV_MAX_TOKENS)
    try:
        g = _full_workload("decode_t64_zipf", list(range(64)))
    finally:
        bm.set_gemv_max_tokens(bm.GEMV_MAX_TOKENS)
    assert int(g["counts"].max()) > 16  # a hot expert serves many tokens


@pytest.mark.parametrize("name", ["prefill_t4096_uniform", "prefill_t4096_zipf"])
def test_prefill_t4096_sampled(name):
    g = _full_workload(name)
    w_ = synth.WORKLOADS[name]
    assert int(g["counts"].sum()) == w_.T * w_.k
    # every output row finite
    assert torch.isfinite(g["out"]).all() and torch.isfinite(g["y"]).all()
