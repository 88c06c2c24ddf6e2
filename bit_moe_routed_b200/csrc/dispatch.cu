// Dispatch: stable counting sort of the T*k (token, slot) pairs by expert
// (dpshk.com article, "核心实现三：多 token 批处理": tokens are grouped per expert so
// that an expert's weights are read once for all tokens routed to it).
//
// One CTA of 32 warps.  Each warp owns a contiguous segment of pair ids, so the
// sorted order within an expert is (warp, position in segment) = ascending pair id.
//   pass 1: per-warp, per-expert counts (match_any groups equal experts of 32 pairs),
//   scan:   per expert, exclusive prefix over warps; then exclusive scan over experts,
//   pass 2: each pair's position = offsets[e] + warp prefix + running count + rank
//           among equal experts in its 32-pair group.
// No atomics decide a position, so the permutation is deterministic.
#include "internal.cuh"
#include "ptx.cuh"

namespace bitmoe {
namespace {

constexpr int kWarps = 32;

__global__ void __launch_bounds__(1024, 1) dispatch_kernel(const int32_t* __restrict__ idx, int P,
                                                           int E, int32_t* __restrict__ counts,
                                                           int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ perm,
                                                           int32_t* __restrict__ pos,
                                                           int* __restrict__ status) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // idx comes from earlier work on the stream
  extern __shared__ int32_t sm[];
  int32_t* cnt = sm;                     // [kWarps][E]
  int32_t* off = sm + kWarps * E;        // [E+1]
  int32_t* wsum = off + E + 1;           // [32] scan scratch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();

  const int seg = (P + kWarps - 1) / kWarps;
  const int beg = min(P, warp * seg), end = min(P, beg + seg);
  const unsigned lt_mask = (1u << lane) - 1u;

  // pass 1: counts per (warp, expert)
  for (int base = beg; base < end; base += 32) {
    const int i = base + lane;
    int e = i < end ? __ldg(idx + i) : -1;
    if (i < end && (e < 0 || e >= E)) {  // out-of-range expert id: flag it, skip the pair
      atomicOr(status, kStatusBadIndex);
      e = -1;
    }
    const bool valid = e >= 0;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (valid && (peers & lt_mask) == 0) cnt[warp * E + e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();

  // per expert: exclusive prefix over warps, totals
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int c = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += c;
    }
    off[e] = run;  // total count for now
  }
  __syncthreads();

  // exclusive scan of the totals over experts (E <= 1024: one value per thread)
  {
    const int e = threadIdx.x;
    const int v = e < E ? off[e] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int ws = wsum[lane];
      int wi = ws;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      wsum[lane] = wi - ws;  // exclusive prefix of the warp sums
      if (lane == 31) off[E] = wi;
    }
    __syncthreads();
    if (e < E) {
      const int excl = wsum[warp] + incl - v;
      counts[e] = v;
      offsets[e] = excl;
      off[e] = excl;
    }
    if (threadIdx.x == 0) offsets[E] = off[E];
  }
  __syncthreads();

  // pass 2: positions
  for (int base = beg; base < end; base += 32) {
    const int i = base + lane;
    int e = i < end ? __ldg(idx + i) : -1;
    if (e >= E) e = -1;
    const bool valid = e >= 0;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (valid) {
      const int p = off[e] + cnt[warp * E + e] + __popc(peers & lt_mask);
      perm[p] = i;
      pos[i] = p;
    }
    __syncwarp();
    if (valid && (peers & lt_mask) == 0) cnt[warp * E + e] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_dispatch(const int32_t* idx, int T, int k, int E, int32_t* counts,
                            int32_t* offsets, int32_t* perm, int32_t* pos, int* status,
                            cudaStream_t s, bool overlap) {
  const size_t smem = sizeof(int32_t) * ((size_t)kWarps * E + E + 1 + 32);
  cudaError_t err = cudaFuncSetAttribute(dispatch_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(dispatch_kernel, dim3(1), dim3(1024), smem, s, overlap, idx, T * k, E, counts, offsets,
                    perm, pos, status);
}

}  // namespace bitmoe
