"""The FFN writes only inside the workspace it is given: a guard region placed right after
a workspace of exactly moe_workspace_size bytes keeps its fill pattern through the whole
layer, for batch sizes that take each tile shape (256-row tiles at T <= 64, 128-row tiles
above) and split tiles between CTAs."""
import pytest
import torch

import synth
from helpers import device_weights

pytestmark = pytest.mark.gpu

bm = pytest.importorskip("bit_moe_routed_b200")

GUARD = 4 << 20


@pytest.mark.parametrize("T", [1, 5, 64, 65, 100])
def test_ffn_stays_inside_workspace(T):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    E, k, d, f = 256, 6, 4096, 2048
    W = device_weights(7100 + T, 0, E, d, f)
    x = synth.gen_x(T, d, seed=7200 + T).cuda()
    s = synth.gen_scores_zipf(T, E, 1.0, seed=7300 + T).cuda()
    n = bm.workspace_size(T, k, E, d, f)
    buf = torch.full((n + GUARD,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[:n]
    idx, gw = bm.route_topk(s, k)
    counts, offsets, perm, pos = bm.dispatch(idx, E)
    y, ysh = bm.expert_ffn(x, k, W, offsets, perm, ws)
    bm.combine(y, ysh, gw, pos)
    bm.forward(x, s, k, W, ws)  # the whole-layer call (one kernel at T = 1)
    bm.sync_status()
    tail = buf[n:]
    bad = int((tail != 0xA5).sum())
    assert bad == 0, f"T={T}: {bad} guard bytes after the workspace were overwritten"
