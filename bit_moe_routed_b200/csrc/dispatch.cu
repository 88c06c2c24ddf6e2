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

// ---------------------------------------------------------------- multi-CTA form
// For large batches the pairs are cut into segments of kSegPairs, one per CTA (8 warps,
// each a contiguous sub-segment).  Kernel 1 writes each CTA's per-expert counts to
// cnt[b][E]; kernel 2 has every CTA rebuild the totals (exclusive scan over experts =
// offsets) and its own base per expert (sum of the counts of the CTAs before it), then
// place its pairs exactly as the one-CTA kernel does: sorted position = offsets[e] + base
// + rank within the segment.  Segments are in pair-id order, so the result is the same
// stable permutation, bit for bit.
constexpr int kSegWarps = 8;
constexpr int kSegPairs = 1024;

__global__ void __launch_bounds__(kSegWarps * 32) dispatch_count_kernel(
    const int32_t* __restrict__ idx, int P, int E, int32_t* __restrict__ cnt,
    int* __restrict__ status) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  extern __shared__ int32_t sm[];  // [E]
  for (int e = threadIdx.x; e < E; e += blockDim.x) sm[e] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int beg = blockIdx.x * kSegPairs, end = min(P, beg + kSegPairs);
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = beg + (threadIdx.x & ~31); base < end; base += blockDim.x) {
    const int i = base + lane;
    int e = i < end ? __ldg(idx + i) : -1;
    if (i < end && (e < 0 || e >= E)) {
      atomicOr(status, kStatusBadIndex);
      e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt_mask) == 0) atomicAdd(&sm[e], __popc(peers));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[(size_t)blockIdx.x * E + e] = sm[e];
}

__global__ void __launch_bounds__(kSegWarps * 32) dispatch_scatter_kernel(
    const int32_t* __restrict__ idx, int P, int E, const int32_t* __restrict__ cnt,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ pos) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // the counts of every segment
  extern __shared__ int32_t sm[];
  int32_t* off = sm;                  // [E+1] offsets, then this CTA's next position per expert
  int32_t* wcnt = sm + E + 1;         // [kSegWarps][E]: the warps' counts, then their prefixes
  int32_t* wsum = wcnt + kSegWarps * E;  // [32] scan scratch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, b = blockIdx.x;
  // totals and this CTA's base per expert, then the exclusive scan of the totals
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    int tot = 0, before = 0;
    if (e < E)
      for (int c = 0; c < G; ++c) {
        const int v = __ldcg(cnt + (size_t)c * E + e);
        before += c < b ? v : 0;
        tot += v;
      }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = lane < kSegWarps ? wsum[lane] : 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
      }
      if (lane < kSegWarps) wsum[lane] = x - v;                 // exclusive per warp
      if (lane == kSegWarps - 1) wsum[kSegWarps] = x;            // this round's total
    }
    __syncthreads();
    const int carry = e0 == 0 ? 0 : off[E];                      // offset of expert e0
    if (e < E) {
      const int excl = carry + wsum[warp] + incl - tot;
      off[e] = excl + before;  // where this CTA's pairs of expert e start
      if (b == 0) {
        counts[e] = tot;
        offsets[e] = excl;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) off[E] = carry + wsum[kSegWarps];
    __syncthreads();
  }
  if (b == 0 && threadIdx.x == 0) offsets[E] = off[E];
  // per-warp counts of this segment, then exclusive prefixes over the warps
  for (int i = threadIdx.x; i < kSegWarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  const int beg = b * kSegPairs, end = min(P, beg + kSegPairs);
  const int sub = (kSegPairs + kSegWarps - 1) / kSegWarps;
  const int wb = min(end, beg + warp * sub), we = min(end, wb + sub);
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = wb; base < we; base += 32) {
    const int i = base + lane;
    int e = i < we ? __ldg(idx + i) : -1;
    if (e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt_mask) == 0) wcnt[warp * E + e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = off[e];
    for (int w = 0; w < kSegWarps; ++w) {
      const int c = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int base = wb; base < we; base += 32) {
    const int i = base + lane;
    int e = i < we ? __ldg(idx + i) : -1;
    if (e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int p = wcnt[warp * E + e] + __popc(peers & lt_mask);
      perm[p] = i;
      pos[i] = p;
    }
    __syncwarp();
    if (e >= 0 && (peers & lt_mask) == 0) wcnt[warp * E + e] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace

size_t dispatch_ws_bytes(int T, int k, int E) {
  const long long P = (long long)T * k;
  return P >= kDispatchMultiMin ? (size_t)((P + kSegPairs - 1) / kSegPairs) * E * 4 : 0;
}

cudaError_t launch_dispatch_multi(const int32_t* idx, int T, int k, int E, int32_t* counts,
                                  int32_t* offsets, int32_t* perm, int32_t* pos, int32_t* cnt,
                                  int* status, cudaStream_t s, bool overlap) {
  const int P = T * k;
  const unsigned G = (unsigned)((P + kSegPairs - 1) / kSegPairs);
  const size_t smem1 = sizeof(int32_t) * (size_t)E;
  const size_t smem2 = sizeof(int32_t) * ((size_t)E + 1 + (size_t)kSegWarps * E + 32);
  cudaError_t err = cudaFuncSetAttribute(dispatch_scatter_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
  if (err != cudaSuccess) return err;
  err = launch_pdl(dispatch_count_kernel, dim3(G), dim3(kSegWarps * 32), smem1, s, overlap, idx, P, E,
                   cnt, status);
  if (err != cudaSuccess) return err;
  return launch_pdl(dispatch_scatter_kernel, dim3(G), dim3(kSegWarps * 32), smem2, s, true, idx, P,
                    E, (const int32_t*)cnt, counts, offsets, perm, pos);
}

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
