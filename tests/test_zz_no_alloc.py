"""moe_expert_ffn_noalloc: the expert FFN for callers that cannot allocate device memory
(its scratch is a fixed array inside the library).  Checked through the C ABI against
moe_expert_ffn with a caller-owned workspace, on two calls in a row with different
inputs, and its size limit is checked on the host."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from helpers import assert_close

pytestmark = pytest.mark.gpu

bm = pytest.importorskip("bit_moe_routed_b200")


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    T, E, k, d, f = 16, 256, 6, 4096, 2048
    W = bm.LayerWeights.from_dict(synth.device_layer_weights(4242, 0, E, d, f))
    for call in range(2):
        x = synth.gen_x(T, d, seed=4300 + call).cuda()
        s = synth.gen_scores_zipf(T, E, 1.0, seed=4400 + call).cuda()
        idx, _ = bm.route_topk(s, k)
        _, offsets, perm, _ = bm.dispatch(idx, E)
        y_ref, ysh_ref = bm.expert_ffn(x, k, W, offsets, perm)
        y, ysh = bm.expert_ffn_noalloc(x, k, W, offsets, perm)
        bm.sync_status()
        assert_close(y.cpu().numpy(), y_ref.cpu().numpy(), f"call {call}: y_routed")
        assert_close(ysh.cpu().numpy(), ysh_ref.cpu().numpy(), f"call {call}: y_shared")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = bm.lib()
    w = bm._Weights(256, 256, 256, 256, 256, 256, 256, 4096, 2048)
    P = ctypes.c_void_p(256)
    rc = L.moe_expert_ffn_noalloc(P, 4096, 6, ctypes.byref(w), P, P, P, P, None)
    assert rc == bm.MOE_ERR_WORKSPACE
    assert b"needs" in L.moe_last_error()
