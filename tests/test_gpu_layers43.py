"""43 independent MoE layers resident in HBM (147.7 GB of FP4 weights and scales), run back
to back at T=1 and T=32 with Zipf(1.0) routing; every layer's output is checked against
the oracle on sampled tokens (weights regenerated on the host for the experts used): the
one token at T=1, four tokens per layer at T=32 (chosen to cover the tiles' edges)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import check_layer, gpu_layer, tile_sample_tokens

pytestmark = pytest.mark.gpu

bm = pytest.importorskip("bit_moe_routed_b200")


@pytest.fixture(scope="module")
def layers():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    torch.cuda.empty_cache()
    w_ = synth.WORKLOADS["layers43_t1"]
    need = w_.layers * synth.expert_bytes(w_.d, w_.f) * (w_.E + 1)
    free, _ = torch.cuda.mem_get_info()
    if free < need + (4 << 30):
        pytest.skip(f"needs {need / 1e9:.1f} GB free, have {free / 1e9:.1f}")
    # both T=1 and T=32 workloads share the layer weights of draw 0 (seed of layer l)
    Ws = [bm.LayerWeights.from_dict(synth.device_layer_weights(w_.seed(l), l, w_.E, w_.d, w_.f))
          for l in range(w_.layers)]
    yield Ws
    del Ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,n_tokens", [("layers43_t1", 1), ("layers43_t32", 4)])
def test_43_layers_back_to_back(layers, name, n_tokens):
    w_ = synth.WORKLOADS[name]
    base = synth.WORKLOADS["layers43_t1"]
    oracle.set_threads(8)
    ws = bm.alloc_workspace(w_.T, w_.k, w_.E, w_.d, w_.f)
    inputs = [synth.gen_layer_inputs(w_, l) for l in range(w_.layers)]
    results = []
    for l in range(w_.layers):  # all layers first, on the device, back to back
        x, s = inputs[l]
        results.append(gpu_layer(x, s, w_.k, layers[l], ws, keep_device=True))
    bm.sync_status()
    for l in range(w_.layers):
        x, s = inputs[l]
        idx, _ = oracle.route_topk(s.numpy(), w_.k)
        tokens = tile_sample_tokens(idx, w_.E, n_tokens, seed=l)
        check_layer(results[l], x, s, w_.k, w_.E, w_.d, w_.f, base.seed(l), l, tokens,
                    f"{name} layer {l}")
