// Top-k routing: one warp per token (tcti.cn post, "DeepSeek-V4-Flash的可能性": each token
// activates 6 of the 256 routed experts).  Each lane holds the scores of experts
// lane, lane+32, ...; k rounds of a warp arg-max pick the winners in descending order
// (equal scores: lower expert index first).  The combine weights are the sigmoids of
// the selected scores renormalised to sum 1, computed in fp32.
#include "internal.cuh"
#include "ptx.cuh"

namespace bitmoe {
namespace {

template <int PER_LANE>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ scores, int T, int E,
                                                   int k, int32_t* __restrict__ idx_out,
                                                   float* __restrict__ w_out) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // scores come from earlier work on the stream
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const float* s = scores + (size_t)warp * E;
  float v[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(s + e) : -INFINITY;
  }
  unsigned taken = 0;  // bit i: v[i] already selected
  float sel_v = 0.f;
  int sel_i = 0;
  for (int j = 0; j < k; ++j) {
    // lane-local best among the not-yet-taken (index order lane + 32 i is ascending in i)
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
      const int e = lane + 32 * i;
      const bool ok = !((taken >> i) & 1u) && e < E;
      if (ok && (v[i] > bv || (v[i] == bv && e < bi))) {
        bv = v[i];
        bi = e;
      }
    }
    // warp arg-max on (value desc, index asc)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) {
      sel_v = bv;
      sel_i = bi;
    }
  }
  // gate weights: sigmoid of the selected scores, renormalised (lanes 0..k-1)
  const float sig = lane < k ? 1.0f / (1.0f + expf(-sel_v)) : 0.0f;
  float sum = sig;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane < k) {
    idx_out[(size_t)warp * k + lane] = sel_i;
    w_out[(size_t)warp * k + lane] = sig / sum;
  }
}

}  // namespace

cudaError_t launch_route_topk(const float* scores, int T, int E, int k, int32_t* idx, float* w,
                              cudaStream_t s, bool overlap) {
  const int warps_per_block = 8;
  const unsigned blocks = (unsigned)((T + warps_per_block - 1) / warps_per_block);
  if (E <= 256)
    return launch_pdl(topk_kernel<8>, dim3(blocks), dim3(256), 0, s, overlap, scores, T, E, k, idx, w);
  if (E <= 512)
    return launch_pdl(topk_kernel<16>, dim3(blocks), dim3(256), 0, s, overlap, scores, T, E, k, idx, w);
  return launch_pdl(topk_kernel<32>, dim3(blocks), dim3(256), 0, s, overlap, scores, T, E, k, idx, w);
}

}  // namespace bitmoe
