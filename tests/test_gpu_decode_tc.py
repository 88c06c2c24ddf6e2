"""The tensor-core single-token layer kernel (decode_tc.cu) against the oracle.

moe_forward at T = 1 runs it where the shapes allow under moe_set_decode_engine(1):
routing, dispatch and the token's codes bit for bit; the re-quantised h under the tie rule
and its fp32 value within the a-priori bound; y, y_shared and out within the bounds of the
parity rules (tests/helpers.py, check_layer).  Also: the choice of form, determinism over
repeated calls, a workspace shared by layers of other shapes (its counters carry an epoch
tag, so a count an earlier call left behind reads as zero), and the CUDA-core form on the
same inputs."""
import numpy as np
import pytest
import torch

import bit_moe_routed_b200 as bm
import synth
from helpers import check_layer, device_weights, gpu_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _engine():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    bm.set_decode_engine(1)
    yield
    bm.set_decode_engine(0)  # the default


def _inputs(E, d, seed, zipf=False):
    x = synth.gen_x(1, d, seed=seed)
    s = synth.gen_scores_zipf(1, E, 1.2, seed + 1) if zipf else synth.gen_scores_uniform(1, E, seed + 1)
    return x, s


@pytest.mark.parametrize("E,k,d,f", [
    (8, 2, 512, 512),       # two K chunks per row block in each phase
    (16, 1, 1024, 512),     # one routed expert
    (64, 8, 1024, 1536),    # f not a power of two: 12 row blocks of h
    (256, 6, 2048, 1024),
    (32, 4, 4096, 1024),    # four TMEM column groups in phase 1
    (1024, 8, 1024, 512),   # top-k over 32 scores per lane
    (64, 32, 512, 512),     # the most experts per token
])
def test_tc_single_token_shapes(E, k, d, f):
    W = device_weights(E + d + f + k, 0, E, d, f)
    assert bm.forward_path(1, k, W) == bm.PATH_SINGLE_TC
    x, s = _inputs(E, d, seed=E + d + f + k)
    g = gpu_layer(x, s, k, W)
    check_layer(g, x, s, k, E, d, f, E + d + f + k, 0, [0], f"tensor cores E={E} k={k} d={d} f={f}")


@pytest.mark.parametrize("zipf", [False, True], ids=["uniform", "zipf"])
def test_tc_decode_t1_full_size(zipf):
    """The decode workload's sizes (256 + 1 experts, top-6, d = 4096, f = 2048)."""
    E, k, d, f = 256, 6, 4096, 2048
    W = device_weights(71, 0, E, d, f)
    x, s = _inputs(E, d, seed=72, zipf=zipf)
    g = gpu_layer(x, s, k, W)
    check_layer(g, x, s, k, E, d, f, 71, 0, [0], "tensor cores, decode_t1 sizes")


def test_tc_forms_and_fallback_shapes():
    """The form each shape takes: the CUDA-core form for engine 0, and for a shape outside
    the tensor-core kernel's limits (f = 2560: three experts' h tiles, 60 KB, do not fit
    beside the stage ring)."""
    W = device_weights(81, 0, 16, 1024, 512)
    assert bm.forward_path(1, 2, W) == bm.PATH_SINGLE_TC
    bm.set_decode_engine(0)
    assert bm.forward_path(1, 2, W) == bm.PATH_SINGLE
    bm.set_decode_engine(1)
    W2 = device_weights(82, 0, 8, 1024, 2560)
    assert bm.forward_path(1, 2, W2) == bm.PATH_SINGLE
    x, s = _inputs(8, 1024, seed=83)
    g = gpu_layer(x, s, 2, W2)
    check_layer(g, x, s, 2, 8, 1024, 2560, 82, 0, [0], "f = 2560 on the CUDA cores")
    with pytest.raises(bm.MoeError):
        bm.set_decode_engine(2)


def test_tc_repeated_calls_are_identical():
    """Every sum runs in a fixed order: three calls give the same bits."""
    E, k, d, f = 256, 6, 4096, 2048
    W = device_weights(91, 0, E, d, f)
    x, s = _inputs(E, d, seed=92)
    ws = bm.alloc_workspace(1, k, E, d, f)
    runs = [gpu_layer(x, s, k, W, ws=ws) for _ in range(3)]
    for r in runs[1:]:
        for name in ("idx", "w", "y", "y_shared", "out", "qh", "sh", "h"):
            assert torch.equal(r[name], runs[0][name]), name
        for name in ("qx", "sx"):  # the single-token kernel writes row 0, the token
            assert torch.equal(r[name][0], runs[0][name][0]), name


def test_tc_workspace_shared_across_shapes():
    """One workspace (sized for the largest layer) serves layers of other shapes in turn:
    the counters another shape left at the same addresses carry an older epoch and read as
    zero, so every call is correct and the first layer's results repeat bit for bit."""
    shapes = [(256, 6, 4096, 2048), (64, 8, 1024, 1536), (16, 2, 2048, 512)]
    size = max(bm.workspace_size(1, k, E, d, f) for E, k, d, f in shapes)
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    first = None
    for rep in range(2):
        for i, (E, k, d, f) in enumerate(shapes):
            W = device_weights(100 + i, 0, E, d, f)
            x, s = _inputs(E, d, seed=110 + i)
            g = gpu_layer(x, s, k, W, ws=ws)
            if rep == 0:
                check_layer(g, x, s, k, E, d, f, 100 + i, 0, [0], f"shared workspace {E, k, d, f}",
                            verbose=False)
                if i == 0:
                    first = g
            elif i == 0:
                for name in ("y", "y_shared", "out", "qh", "sh"):
                    assert torch.equal(g[name], first[name]), name


def test_tc_and_cuda_core_forms_agree_within_bounds():
    """Both forms of the kernel on the same token meet the oracle's bounds; they share the
    routing, dispatch and token codes bit for bit."""
    E, k, d, f = 256, 6, 4096, 2048
    W = device_weights(121, 0, E, d, f)
    x, s = _inputs(E, d, seed=122)
    a = gpu_layer(x, s, k, W)
    bm.set_decode_engine(0)
    b = gpu_layer(x, s, k, W)
    for name in ("idx", "w", "counts", "offsets", "perm", "pos"):
        assert torch.equal(a[name], b[name]), name
    assert torch.equal(a["qx"][0], b["qx"][0]) and torch.equal(a["sx"][0], b["sx"][0])
    check_layer(a, x, s, k, E, d, f, 121, 0, [0], "tensor-core form")
    check_layer(b, x, s, k, E, d, f, 121, 0, [0], "CUDA-core form")
    rel = (a["out"] - b["out"]).norm() / b["out"].norm()
    assert float(rel) < 1e-5, float(rel)


def test_tc_zero_token():
    """An all-zero token: every activation block has scale 1 and zero codes, so h and every
    output are exactly zero."""
    E, k, d, f = 64, 4, 1024, 512
    W = device_weights(131, 0, E, d, f)
    x = torch.zeros((1, d), dtype=torch.bfloat16)
    s = synth.gen_scores_uniform(1, E, 132)
    g = gpu_layer(x, s, k, W)
    check_layer(g, x, s, k, E, d, f, 131, 0, [0], "zero token")
    assert float(g["out"].abs().max()) == 0.0
    assert np.all(g["sh"].numpy()[: k + 1] == 1.0)
