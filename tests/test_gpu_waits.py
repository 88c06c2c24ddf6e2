"""Failure detection without a GPU fault: the FFN kernels bound every wait by a
%globaltimer limit.  A 1 ns limit makes the first wait that is not already satisfied run
out; the kernel must record MOE_ERR_TIMEOUT, release TMEM (tile kernels), drain its
copies and return, leaving the context usable for the next (normal) call.  The tile
kernels (T = 8) run with the tiny limit.  The single-token kernels wait only on their own
TMA stages, and one try_wait usually outlasts a stage's copy, so there a tiny limit may or
may not run out; their timeout path is exercised deterministically by the test stall
(moe_set_test_stall), a wait on a barrier that nothing completes."""
import numpy as np
import pytest
import torch

import synth
from helpers import check_layer, device_weights, gpu_layer

pytestmark = pytest.mark.gpu

bm = pytest.importorskip("bit_moe_routed_b200")


def test_wait_limit_expiry_is_reported_and_recoverable():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    T, E, k, d, f = 8, 16, 2, 512, 256  # tcgen05 tile kernels
    x = synth.gen_x(T, d, seed=501)
    s = synth.gen_scores_uniform(T, E, seed=502)
    W = device_weights(503, 0, E, d, f)
    bm.sync_status()  # clean start
    bm.set_wait_limit_ns(1)
    try:
        bm.forward(x.cuda(), s.cuda(), k, W)
        with pytest.raises(bm.MoeError) as ei:
            bm.sync_status()
        assert ei.value.code == bm.MOE_ERR_TIMEOUT
    finally:
        bm.set_wait_limit_ns(0)  # default limit
    bm.sync_status()  # the status word was cleared by the report
    g = gpu_layer(x, s, k, W)
    check_layer(g, x, s, k, E, d, f, 503, 0, list(range(T)), "after timeout")


def test_gemv_tiny_wait_limit_reports_or_completes():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    T, E, k, d, f = 1, 64, 6, 4096, 2048  # single-token GEMV kernels, decode-sized rows
    x = synth.gen_x(T, d, seed=511)
    s = synth.gen_scores_uniform(T, E, seed=512)
    W = device_weights(513, 0, E, d, f)
    bm.sync_status()
    bm.set_wait_limit_ns(1)
    try:
        r = bm.forward(x.cuda(), s.cuda(), k, W)
        try:
            bm.sync_status()
            timed_out = False
        except bm.MoeError as e:
            assert e.code == bm.MOE_ERR_TIMEOUT
            timed_out = True
        g = {kk: v.cpu() for kk, v in r.items()}
    finally:
        bm.set_wait_limit_ns(0)
    if not timed_out:
        check_layer(g, x, s, k, E, d, f, 513, 0, [0], "tiny limit, no timeout")
    bm.sync_status()
    g = gpu_layer(x, s, k, W)
    check_layer(g, x, s, k, E, d, f, 513, 0, [0], "after the tiny limit")


@pytest.mark.parametrize("engine", [0, 1], ids=["cuda_cores", "tensor_cores"])
def test_single_token_stall_times_out_and_recovers(engine):
    """The test stall makes one warp's bounded wait run out on every call: the status must
    report MOE_ERR_TIMEOUT each time, and the next normal call must be correct (both forms
    of the single-token kernel)."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    bm.set_decode_engine(engine)
    T, E, k, d, f = 1, 64, 6, 4096, 2048
    x = synth.gen_x(T, d, seed=521)
    s = synth.gen_scores_uniform(T, E, seed=522)
    W = device_weights(523, 0, E, d, f)
    bm.sync_status()
    bm.set_wait_limit_ns(20_000_000)  # 20 ms
    bm.set_test_stall(True)
    try:
        for _ in range(2):
            bm.forward(x.cuda(), s.cuda(), k, W)
            with pytest.raises(bm.MoeError) as ei:
                bm.sync_status()
            assert ei.value.code == bm.MOE_ERR_TIMEOUT
    finally:
        bm.set_test_stall(False)
        bm.set_wait_limit_ns(0)
    bm.sync_status()
    try:
        g = gpu_layer(x, s, k, W)
    finally:
        bm.set_decode_engine(0)  # the default
    check_layer(g, x, s, k, E, d, f, 523, 0, [0], "after the stall")
