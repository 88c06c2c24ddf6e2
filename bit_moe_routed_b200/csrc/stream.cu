// Routed experts streamed from host memory into an HBM expert cache (NEXT-4, one GPU).
//
// The pages' central systems theme is running a model whose routed experts do not fit the
// accelerator: they stay in host RAM (tcti.cn post, "DeepSeek-V4-Flash的可能性": routed
// experts in host memory, attention and the shared expert resident) and are read as they
// are needed, under an LRU share (dpshk.com article, "核心实现一": expert streaming).  Here
// the routed experts live in pinned, device-mapped host memory; an HBM cache of S slots
// holds the recently used ones (slot S: the shared expert, always resident), and one
// token's layer runs as three kernels on the stream, with no host round trip:
//   route    the top-k of the scores (topk_kernel) into the call's topk_idx;
//   cache    one thread applies the LRU policy: the selected experts (ascending id) that
//            are resident are marked used; each one that is not takes the least recently
//            used slot not holding an expert of this token (empty slots first, ties to
//            the lower slot), whose expert is evicted; the (expert, slot) fills are
//            listed;
//   fetch    every CTA copies its share of the listed experts' codes and scales from host
//            memory (16-byte loads over PCIe) into their slots;
// then the single-token layer kernel reads the weights through the expert -> slot table.
// Results equal those of moe_forward on resident weights bit for bit (the same kernel on
// the same bytes).
#include "internal.cuh"
#include "ptx.cuh"

namespace bitmoe {
namespace {

__global__ void cache_kernel(const int32_t* __restrict__ idx, int k, int S,
                             int32_t* __restrict__ slot_of, int32_t* __restrict__ expert_of,
                             long long* __restrict__ last_use, long long* __restrict__ clock,
                             int32_t* __restrict__ fetch, long long* __restrict__ stats,
                             int* status) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // idx comes from the routing kernel
  if (threadIdx.x != 0) return;
  int sel[32];
  int n = 0;
  for (int j = 0; j < k; ++j) {  // the selected experts in ascending id, once each
    const int e = idx[j];
    int pos = n;
    bool dup = false;
    for (int i = 0; i < n; ++i) dup |= sel[i] == e;
    if (dup) continue;
    while (pos > 0 && sel[pos - 1] > e) {
      sel[pos] = sel[pos - 1];
      --pos;
    }
    sel[pos] = e;
    ++n;
  }
  const long long now = *clock + 1;
  *clock = now;
  int hits = 0, nf = 0;
  for (int i = 0; i < n; ++i) {
    const int s = slot_of[sel[i]];
    if (s >= 0) {
      last_use[s] = now;
      ++hits;
    }
  }
  for (int i = 0; i < n; ++i) {
    const int e = sel[i];
    if (slot_of[e] >= 0) continue;
    int best = -1;
    for (int s = 0; s < S; ++s) {
      const int ex = expert_of[s];
      bool cur = false;
      for (int q = 0; q < n; ++q) cur |= ex == sel[q];
      if (cur) continue;
      if (best < 0 || last_use[s] < last_use[best]) best = s;
    }
    if (best < 0) {  // fewer slots than selected experts (the host rejects such caches)
      atomicOr(status, kStatusBadIndex);
      break;
    }
    if (expert_of[best] >= 0) slot_of[expert_of[best]] = -1;
    expert_of[best] = e;
    slot_of[e] = best;
    last_use[best] = now;
    fetch[1 + 2 * nf] = e;
    fetch[2 + 2 * nf] = best;
    ++nf;
  }
  fetch[0] = nf;
  stats[0] += hits;
  stats[1] += nf;
}

struct FetchParams {
  const uint8_t* src[6];  // host arrays: gate codes, gate scales, up codes, up scales, down ...
  uint8_t* dst[6];        // slot arrays, same order
  long long bytes[6];     // bytes per expert of each array (multiples of 16)
  const int32_t* fetch;
};

__global__ void __launch_bounds__(256) fetch_kernel(const FetchParams p) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // the fill list comes from the cache kernel
  const int nf = p.fetch[0];
  long long per = 0;  // 16-byte vectors per expert over the six arrays
  for (int a = 0; a < 6; ++a) per += p.bytes[a] / 16;
  const long long total = per * nf;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long v0 = (long long)blockIdx.x * blockDim.x + threadIdx.x; v0 < total; v0 += 4 * stride) {
    uint4 buf[4];
    uint4* dst[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // four loads in flight before any store
      const long long v = v0 + u * stride;
      dst[u] = nullptr;
      if (v < total) {
        const int f = (int)(v / per);
        long long r = v - (long long)f * per;
        int a = 0;
        while (r >= p.bytes[a] / 16) {
          r -= p.bytes[a] / 16;
          ++a;
        }
        const int e = p.fetch[1 + 2 * f], s = p.fetch[2 + 2 * f];
        const uint4* src = reinterpret_cast<const uint4*>(p.src[a] + (long long)e * p.bytes[a]) + r;
        buf[u] = *src;
        dst[u] = reinterpret_cast<uint4*>(p.dst[a] + (long long)s * p.bytes[a]) + r;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (dst[u]) *dst[u] = buf[u];
  }
}

}  // namespace

cudaError_t launch_cache(const int32_t* idx, int k, int S, int32_t* slot_of, int32_t* expert_of,
                         long long* last_use, long long* clock, int32_t* fetch, long long* stats,
                         int* status, cudaStream_t s) {
  return launch_pdl(cache_kernel, dim3(1), dim3(32), 0, s, true, idx, k, S, slot_of, expert_of,
                    last_use, clock, fetch, stats, status);
}

cudaError_t launch_fetch(const uint8_t* const src[6], uint8_t* const dst[6],
                         const long long bytes[6], const int32_t* fetch, int num_sms,
                         cudaStream_t s) {
  FetchParams p;
  for (int a = 0; a < 6; ++a) {
    p.src[a] = src[a];
    p.dst[a] = dst[a];
    p.bytes[a] = bytes[a];
  }
  p.fetch = fetch;
  return launch_pdl(fetch_kernel, dim3((unsigned)(num_sms * 4)), dim3(256), 0, s, true, p);
}

}  // namespace bitmoe
