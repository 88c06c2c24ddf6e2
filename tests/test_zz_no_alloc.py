"""moe_expert_ffn_noalloc: the expert FFN for callers that cannot allocate device memory
when they run the layer (an engine plugin handed no workspace, a serving loop that must
not call cudaMalloc because it can synchronise the device); its scratch is a fixed array
inside the library.

Checked through the C ABI against moe_expert_ffn with a caller-owned workspace, on two
calls in a row with different inputs, at one token (the single-token kernels, whose fp32
hidden state lives in the scratch), 16 tokens (small tiles) and 72 tokens (the largest
batch the scratch holds at d = 4096, f = 2048, k = 6, E = 256; its stream-K partial slots
sit near the end of the array).  The kernels are deterministic, so the two entry points
must agree bit for bit.  The single-token call is also checked against the oracle, and the
size limit on the host (no GPU needed)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import check_layer

bm = pytest.importorskip("bit_moe_routed_b200")

E, K_, D, F = 256, 6, 4096, 2048


@pytest.fixture(scope="module")
def weights():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    W = bm.LayerWeights.from_dict(synth.device_layer_weights(4242, 0, E, D, F))
    yield W
    del W
    torch.cuda.empty_cache()


@pytest.mark.gpu
@pytest.mark.parametrize("T", [1, 16, 72])
def test_noalloc_matches_workspace_entry_point_on_two_calls(weights, T):
    assert bm.workspace_size(T, K_, E, D, F) <= bm.MOE_NOALLOC_SCRATCH_BYTES
    for call in range(2):
        x = synth.gen_x(T, D, seed=4300 + 10 * T + call)
        s = synth.gen_scores_zipf(T, E, 1.0, seed=4400 + 10 * T + call)
        xd, sd = x.cuda(), s.cuda()
        idx, gw = bm.route_topk(sd, K_)
        counts, offsets, perm, pos = bm.dispatch(idx, E)
        ws = bm.alloc_workspace(T, K_, E, D, F)
        y_ref, ysh_ref = bm.expert_ffn(xd, K_, weights, offsets, perm, ws)
        y, ysh = bm.expert_ffn_noalloc(xd, K_, weights, offsets, perm)
        bm.sync_status()
        assert torch.equal(y, y_ref), f"T={T} call {call}: y_routed differs"
        assert torch.equal(ysh, ysh_ref), f"T={T} call {call}: y_shared differs"
        if T == 1:  # the no-allocation result against the oracle
            out = bm.combine(y, ysh, gw, pos)
            g = dict(idx=idx, w=gw, counts=counts, offsets=offsets, perm=perm, pos=pos, y=y,
                     y_shared=ysh, out=out)
            g.update(bm.workspace_views(ws, T, K_, E, D, F))
            bm.sync_status()
            experts = {e: synth.host_expert(4242, 0, e, D, F)
                       for e in set(idx.cpu().numpy().ravel().tolist()) | {E}}
            check_layer(g, x, s, K_, E, D, F, 4242, 0, [0], f"noalloc T=1 call {call}",
                        experts=experts)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Host-side check before any launch: no GPU needed."""
    L = bm.lib()
    assert bm.workspace_size(72, K_, E, D, F) <= bm.MOE_NOALLOC_SCRATCH_BYTES
    assert bm.workspace_size(73, K_, E, D, F) > bm.MOE_NOALLOC_SCRATCH_BYTES
    w = bm._Weights(256, 256, 256, 256, 256, 256, E, D, F)
    P = ctypes.c_void_p(256)
    for T in (73, 4096):
        rc = L.moe_expert_ffn_noalloc(P, T, K_, ctypes.byref(w), P, P, P, P, None)
        assert rc == bm.MOE_ERR_WORKSPACE
        assert b"needs" in L.moe_last_error()
