// Router scores: scores[t][e] = x[t] . W_router[e] over bf16 inputs with fp32 sums, the step
// before top-k (dpshk.com article, "核心实现一": the router decides each token's experts
// from its hidden state).
//
// A CTA computes one tile of 16 tokens x 8 experts: the M and N of mma.sync m16n8k16 (bf16
// in, fp32 accumulate; every bf16 x bf16 product is exact in fp32).  Its 8 warps take the
// 128-wide K chunks round-robin; each chunk is summed from a fresh accumulator (8 MMAs)
// and added to the warp's running total, and the 8 warp totals are added in warp order,
// so the result does not depend on timing and every product meets at most 128 + K/128 + 8
// roundings.  Fragments come straight from global memory (x rows and W rows are read
// 4 bytes per lane; the tile is small and both stay in L1/L2).
#include "internal.cuh"
#include "ptx.cuh"

namespace bitmoe {
namespace {

constexpr int kRtWarps = 8;

__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3},"
      " {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kRtWarps * 32) router_kernel(const uint16_t* __restrict__ x,
                                                               const uint16_t* __restrict__ w,
                                                               int T, int d, int E,
                                                               float* __restrict__ scores) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // x comes from earlier work on the stream
  __shared__ float part[kRtWarps][16][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int t0 = blockIdx.x * 16, e0 = blockIdx.y * 8;
  // rows of this lane: tokens t0+g, t0+g+8 (A) and expert e0+g (B); out-of-range rows are 0
  const bool ta = t0 + g < T, tb = t0 + g + 8 < T, ew = e0 + g < E;
  const uint32_t* xa = reinterpret_cast<const uint32_t*>(x + (size_t)(ta ? t0 + g : 0) * d);
  const uint32_t* xb = reinterpret_cast<const uint32_t*>(x + (size_t)(tb ? t0 + g + 8 : 0) * d);
  const uint32_t* wr = reinterpret_cast<const uint32_t*>(w + (size_t)(ew ? e0 + g : 0) * d);
  float tot[4] = {0.f, 0.f, 0.f, 0.f};
  for (int c = warp; c < d / 128; c += kRtWarps) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int k2 = (128 * c + 16 * s) / 2 + t;  // 32-bit word of elements k + 2t, k + 2t + 1
      const uint32_t a0 = ta ? __ldg(xa + k2) : 0u, a2 = ta ? __ldg(xa + k2 + 4) : 0u;
      const uint32_t a1 = tb ? __ldg(xb + k2) : 0u, a3 = tb ? __ldg(xb + k2 + 4) : 0u;
      const uint32_t b0 = ew ? __ldg(wr + k2) : 0u, b1 = ew ? __ldg(wr + k2 + 4) : 0u;
      mma_bf16(acc, a0, a1, a2, a3, b0, b1);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) tot[i] += acc[i];
  }
  // acc[0..1]: token g, experts 2t, 2t+1; acc[2..3]: token g+8
  part[warp][g][2 * t] = tot[0];
  part[warp][g][2 * t + 1] = tot[1];
  part[warp][g + 8][2 * t] = tot[2];
  part[warp][g + 8][2 * t + 1] = tot[3];
  __syncthreads();
  if (threadIdx.x < 128) {
    const int tok = threadIdx.x >> 3, ex = threadIdx.x & 7;
    float s = part[0][tok][ex];
    for (int ww = 1; ww < kRtWarps; ++ww) s += part[ww][tok][ex];
    if (t0 + tok < T && e0 + ex < E) scores[(size_t)(t0 + tok) * E + e0 + ex] = s;
  }
}

}  // namespace

cudaError_t launch_router(const uint16_t* x, const uint16_t* w, int T, int d, int E, float* scores,
                          cudaStream_t s, bool overlap) {
  const dim3 grid((unsigned)((T + 15) / 16), (unsigned)((E + 7) / 8));
  return launch_pdl(router_kernel, grid, dim3(kRtWarps * 32), 0, s, overlap, x, w, T, d, E, scores);
}

}  // namespace bitmoe
