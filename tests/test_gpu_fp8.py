"""GPU parity of the FP8 x FP8 GEMM (moe_fp8_gemm) and of the FP8-weight shared expert
(moe_shared_expert_fp8) against the oracle (oracle_fp8_gemm and the FP8 codec of the
expert FFN, pinned in tests/test_oracle_fp8.py).

Bounds are a-priori, as for the FP4 path: every product of two e4m3 values is exact in
fp32; a product meets at most 127 roundings inside its 128-element block (the tensor
core's sum), one for the weight scale, one fused multiply-add per block into the task's
sum and at most K/512 more when the tasks' partials are added, so
|C_gpu - C| <= D * 2^-23 * sum_k |A_k B_k| sa sb with D = 130 + K/128 + K/512."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import HStats, U23, assert_close, assert_within, check_h_codes, h_bound_from

pytestmark = pytest.mark.gpu
bm = pytest.importorskip("bit_moe_routed_b200")


def depth8(K):
    return 130 + K // 128 + K // 512


def fp8_bound(A, sa, B, sb):
    K = A.shape[1]
    return 1.01 * depth8(K) * U23 * oracle.fp8_gemm(A & 0x7F, sa, B & 0x7F, sb)


@pytest.mark.parametrize("M,N,K", [(1, 2048, 4096), (1, 4096, 2048), (3, 256, 512),
                                   (8, 1024, 1024), (17, 512, 2048), (64, 256, 4096)])
def test_fp8_gemm_matches_oracle(M, N, K):
    ex = synth.host_expert_fp8(M + N + K, 0, K, N)  # gate [N][K], scales [N/128][K/128]
    B, sb = ex["gate"], ex["gate_scales"]
    x = synth.gen_x(M, K, seed=M * 31 + K)
    A, sa = oracle.act_quant(x)
    C = bm.fp8_gemm(torch.from_numpy(A).cuda(), torch.from_numpy(sa).cuda(),
                    torch.from_numpy(B).cuda(), torch.from_numpy(sb).cuda())
    bm.sync_status()
    ref = oracle.fp8_gemm(A, sa, B, sb)
    worst = assert_within(C.cpu().numpy(), ref, fp8_bound(A, sa, B, sb), f"fp8_gemm {M}x{N}x{K}")
    rel, mabs = assert_close(C.cpu().numpy(), ref, f"fp8_gemm {M}x{N}x{K}")
    print(f"FP8GEMM M={M} N={N} K={K}: worst err/bound {worst:.2e}, rel-L2 {rel:.2e}")


def test_fp8_gemm_repeated_calls_agree_and_reuse_the_workspace():
    M, N, K = 5, 512, 1024
    ex = synth.host_expert_fp8(3, 0, K, N)
    A, sa = oracle.act_quant(synth.gen_x(M, K, seed=9))
    args = [torch.from_numpy(a).cuda() for a in (A, sa, ex["gate"], ex["gate_scales"])]
    ws = torch.empty(int(bm.lib().moe_fp8_gemm_workspace_size(M, N, K)), dtype=torch.uint8,
                     device="cuda")
    c1 = bm.fp8_gemm(*args, ws=ws).clone()
    c2 = bm.fp8_gemm(*args, ws=ws)
    bm.sync_status()
    assert torch.equal(c1, c2)


@pytest.mark.parametrize("T,d,f", [(1, 4096, 2048), (4, 2048, 1024), (64, 1024, 512)])
def test_shared_expert_fp8_matches_oracle(T, d, f):
    seed = 100 + T
    host = synth.host_expert_fp8(seed, 0, d, f)
    dev = bm.Fp8Expert.from_dict(synth.device_expert_fp8(seed, 0, d, f))
    x = synth.gen_x(T, d, seed=seed + 1)
    n = int(bm.lib().moe_shared_expert_fp8_workspace_size(T, d, f))
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    y = bm.shared_expert_fp8(x.cuda(), dev, ws=ws)
    views = {k: v.clone().cpu() for k, v in bm.shared_expert_fp8_views(ws, T, d, f).items()}
    bm.sync_status()
    y = y.cpu().numpy()
    # the device weights are the host ones
    assert torch.equal(dev.gate.cpu(), torch.from_numpy(host["gate"]))
    assert torch.equal(dev.down_scales.cpu(), torch.from_numpy(host["down_scales"]))
    qx, sx = oracle.act_quant(x)
    assert np.array_equal(views["qx"].numpy(), qx) and np.array_equal(views["sx"].numpy(), sx)
    ex = type("Fp8Expert", (), {})()
    ex.codec = oracle.FP8
    for m in ("gate", "up", "down"):
        setattr(ex, f"{m}_codes", host[m])
        setattr(ex, f"{m}_scales", host[f"{m}_scales"])
    g = oracle.fp8_gemm(qx, sx, host["gate"], host["gate_scales"])
    u = oracle.fp8_gemm(qx, sx, host["up"], host["up_scales"])
    ag = oracle.fp8_gemm(qx & 0x7F, sx, host["gate"] & 0x7F, host["gate_scales"])
    au = oracle.fp8_gemm(qx & 0x7F, sx, host["up"] & 0x7F, host["up_scales"])
    stats = HStats()
    h_worst = 0.0
    for t in range(T):
        yo, hq_o, hs_o, hf_o = oracle.expert_ffn_h(ex, d, f, qx[t:t + 1], sx[t:t + 1])
        B = h_bound_from(g[t], u[t], ag[t], au[t], depth8(d))
        h_worst = max(h_worst, assert_within(views["h"].numpy()[t], hf_o[0], B + 2 * U23 * np.abs(hf_o[0]),
                                             f"token {t}: fp32 h"))
        check_h_codes(views["qh"].numpy()[t], views["sh"].numpy()[t], hq_o[0], hs_o[0], hf_o[0],
                      ex, d, None, stats, f"token {t}", bound_fn=lambda rows, B=B: B[rows])
    qh, sh = views["qh"].numpy(), views["sh"].numpy()
    yr = oracle.fp8_gemm(qh, sh, host["down"], host["down_scales"])
    yb = fp8_bound(qh, sh, host["down"], host["down_scales"])
    y_worst = assert_within(y, yr, yb, "y_shared")
    rel, mabs = assert_close(y, yr, "y_shared")
    print(f"FP8SHARED T={T} d={d} f={f}: {stats.line()} | fp32 h worst err/bound {h_worst:.2e}"
          f" | y vs oracle on the GPU's h codes: rel-L2 {rel:.2e}, worst err/bound {y_worst:.2e}")
