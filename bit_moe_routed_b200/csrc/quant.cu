// Activation quantisation (tcti.cn post, "补齐软件栈缺失": act_quant feeds the FP8
// activations of fp4_gemm) fused with the gather of the expert FFN's input rows, and
// the token-tile plan of the FFN kernels.
//
// Row r of the output takes token perm[r] / k for r < P (routed pairs in expert-sorted
// order) and token r - P for P <= r < P + T (shared expert), so every expert's input
// rows are contiguous and the FFN reads them with plain 2-D TMA boxes.
// Per 128-element block: s = amax / 448 (fp32, IEEE divide; 1 if amax == 0),
// q = e4m3(x / s), round to nearest even, saturating.  8 threads share a block; each
// holds 16 consecutive bf16 values (two 16-byte loads) and writes 16 code bytes.
#include "internal.cuh"
#include "ptx.cuh"

namespace bitmoe {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Token tiles: expert e (e < E: routed group offsets[e]..offsets[e+1]; e == E: the T
// shared rows) is cut into ceil(n / nmax) tiles of roundup16(ceil(n / ntiles)) rows,
// the last one shorter.  One warp computes the per-expert tile counts and their scan.
__device__ void write_plan(const int32_t* __restrict__ offsets, int E, int T, int P, int nmax,
                           int32_t* __restrict__ plan) {
  const int lane = threadIdx.x & 31;
  int32_t* ttbase = plan;
  int32_t* tiles = plan + E + 2;
  const int per = (E + 1 + 31) / 32;  // experts per lane, contiguous
  const int e0 = lane * per;
  int local = 0;
  for (int e = e0; e < min(E + 1, e0 + per); ++e) {
    const int n = e < E ? offsets[e + 1] - offsets[e] : T;
    local += (n + nmax - 1) / nmax;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  int base = incl - local;
  for (int e = e0; e < min(E + 1, e0 + per); ++e) {
    const int n = e < E ? offsets[e + 1] - offsets[e] : T;
    const int row = e < E ? offsets[e] : P;
    const int nt = (n + nmax - 1) / nmax;
    ttbase[e] = base;
    if (nt > 0) {
      const int step = (((n + nt - 1) / nt) + 15) / 16 * 16;
      for (int i = 0; i < nt; ++i) {
        tiles[2 * (base + i)] = row + i * step;
        tiles[2 * (base + i) + 1] = min(step, n - i * step);
      }
    }
    base += nt;
  }
  if (lane == 31) ttbase[E + 1] = incl;
}

// Active experts of a single token for the GEMV path: routed experts with a row, in
// ascending id, then the shared expert.  plan[0] = count, then (expert, row) pairs.
__device__ void write_gemv_plan(const int32_t* __restrict__ offsets, int E,
                                int32_t* __restrict__ plan) {
  const int lane = threadIdx.x & 31;
  const int per = (E + 31) / 32;
  const int e0 = lane * per, e1 = min(E, e0 + per);
  int local = 0;
  for (int e = e0; e < e1; ++e) local += offsets[e + 1] > offsets[e] ? 1 : 0;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  int i = incl - local;
  for (int e = e0; e < e1; ++e) {
    if (offsets[e + 1] > offsets[e]) {
      plan[1 + 2 * i] = e;
      plan[2 + 2 * i] = offsets[e];
      ++i;
    }
  }
  if (lane == 31) {
    plan[1 + 2 * incl] = E;
    plan[2 + 2 * incl] = -1;
    plan[0] = incl + 1;
  }
}

// Slots of the batched FP4 GEMV: every expert's rows (routed experts with a group, in
// ascending id, then the shared expert's T rows) cut into slots of at most kBgSlotTokens
// rows.  plan[0] = slots, then (expert, first row, rows) per slot.
__device__ void write_slot_plan(const int32_t* __restrict__ offsets, int E, int T, int P,
                                int32_t* __restrict__ plan) {
  const int lane = threadIdx.x & 31;
  const int per = (E + 1 + 31) / 32;
  const int e0 = lane * per, e1 = min(E + 1, e0 + per);
  int local = 0;
  for (int e = e0; e < e1; ++e) {
    const int n = e < E ? offsets[e + 1] - offsets[e] : T;
    local += (n + kBgSlotTokens - 1) / kBgSlotTokens;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  int i = incl - local;
  for (int e = e0; e < e1; ++e) {
    const int n = e < E ? offsets[e + 1] - offsets[e] : T;
    const int row = e < E ? offsets[e] : P;
    for (int c = 0; c < n; c += kBgSlotTokens, ++i) {
      plan[1 + 3 * i] = e;
      plan[2 + 3 * i] = row + c;
      plan[3 + 3 * i] = min(kBgSlotTokens, n - c);
    }
  }
  if (lane == 31) plan[0] = incl;
}

__global__ void __launch_bounds__(256) quant_rows_kernel(
    const uint16_t* __restrict__ x, int T, int k, int d, const int32_t* __restrict__ perm, int P,
    uint8_t* __restrict__ q, float* __restrict__ s, const int32_t* __restrict__ offsets, int E,
    int nmax, int32_t* __restrict__ plan, int* __restrict__ counters, size_t n_counters,
    int* __restrict__ status, int plan_mode) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // x, perm, offsets, and the counters the previous FFN launch used
  const int R = P + T;
  const int r = blockIdx.x;
  // the FFN kernels' stream-K counters start every launch at zero
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_counters;
       i += (size_t)gridDim.x * blockDim.x)
    counters[i] = 0;
  if (r == R) {  // the plan block
    if (threadIdx.x < 32) {
      if (plan_mode == 1) write_gemv_plan(offsets, E, plan);
      else if (plan_mode == 2) write_slot_plan(offsets, E, T, P, plan);
      else write_plan(offsets, E, T, P, nmax, plan);
    }
    return;
  }
  int t = r < P ? perm[r] / k : r - P;
  bool ok = t >= 0 && t < T;
  if (!ok && threadIdx.x == 0) atomicOr(status, kStatusBadIndex);
  const uint16_t* xr = x + (size_t)(ok ? t : 0) * d;
  // every lane of a warp runs the same number of iterations (full-mask shuffles);
  // a group of 8 lanes (one 128-block) is either wholly inside the row or wholly past it
  const int lane16 = (threadIdx.x & 31) * 16;
  for (int c0 = threadIdx.x * 16; c0 - lane16 < d; c0 += blockDim.x * 16) {
    const bool act = c0 < d;
    uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
    if (act && ok) {
      a = *reinterpret_cast<const uint4*>(xr + c0);
      b = *reinterpret_cast<const uint4*>(xr + c0 + 8);
    }
    const float v[16] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                         bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w),
                         bf16_lo(b.x), bf16_hi(b.x), bf16_lo(b.y), bf16_hi(b.y),
                         bf16_lo(b.z), bf16_hi(b.z), bf16_lo(b.w), bf16_hi(b.w)};
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    // the 8 threads of one 128-block are lanes 8j..8j+7 of a warp
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    const float sc = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
    uint32_t packed[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t lo = ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i], sc), __fdiv_rn(v[4 * i + 1], sc));
      const uint16_t hi =
          ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i + 2], sc), __fdiv_rn(v[4 * i + 3], sc));
      packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    if (act) {
      *reinterpret_cast<uint4*>(q + (size_t)r * d + c0) =
          make_uint4(packed[0], packed[1], packed[2], packed[3]);
      if ((threadIdx.x & 7) == 0) s[(size_t)r * (d / 128) + c0 / 128] = sc;
    }
  }
}

// The inverse of the dispatch's permutation: ipos[perm[r]] = r, the row of each (token,
// choice) pair in expert-sorted order.  A value outside [0, P) is flagged and skipped.
__global__ void __launch_bounds__(256) invperm_kernel(const int32_t* __restrict__ perm, int P,
                                                      int32_t* __restrict__ ipos,
                                                      int* __restrict__ status) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // perm comes from the dispatch
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < P; r += gridDim.x * blockDim.x) {
    const int p = perm[r];
    if (p >= 0 && p < P) ipos[p] = r;
    else atomicOr(status, kStatusBadIndex);
  }
}

// The activation rows in expert-sorted order, one block per token: the token is quantised
// once, as in quant_rows_kernel (s = amax / 448, IEEE divide, 1 if amax = 0; q = e4m3(x / s)
// rounded to nearest even), and its codes and scales go to its k routed rows ipos[t*k + j]
// and to its shared-expert row P + t.  The plan block and the counters as in
// quant_rows_kernel.
__global__ void __launch_bounds__(256) quant_tokens_kernel(
    const uint16_t* __restrict__ x, int T, int k, int d, const int32_t* __restrict__ ipos,
    uint8_t* __restrict__ q, float* __restrict__ s, const int32_t* __restrict__ offsets, int E,
    int nmax, int32_t* __restrict__ plan, int* __restrict__ counters, size_t n_counters,
    int* __restrict__ status, int plan_mode) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // x, ipos, offsets, and the counters the previous FFN launch used
  const int P = T * k;
  const int t = blockIdx.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_counters;
       i += (size_t)gridDim.x * blockDim.x)
    counters[i] = 0;
  if (t == T) {  // the plan block
    if (threadIdx.x < 32) {
      if (plan_mode == 2) write_slot_plan(offsets, E, T, P, plan);
      else write_plan(offsets, E, T, P, nmax, plan);
    }
    return;
  }
  // the token's rows: k routed (from the inverse permutation), then its shared-expert row
  __shared__ int rows[33];
  if (threadIdx.x <= k) {
    int r = threadIdx.x < k ? ipos[(size_t)t * k + threadIdx.x] : P + t;
    if (r < 0 || r >= P + T) {
      atomicOr(status, kStatusBadIndex);
      r = -1;
    }
    rows[threadIdx.x] = r;
  }
  __syncthreads();
  const uint16_t* xr = x + (size_t)t * d;
  const int lane16 = (threadIdx.x & 31) * 16;
  for (int c0 = threadIdx.x * 16; c0 - lane16 < d; c0 += blockDim.x * 16) {
    const bool act = c0 < d;
    uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
    if (act) {
      a = *reinterpret_cast<const uint4*>(xr + c0);
      b = *reinterpret_cast<const uint4*>(xr + c0 + 8);
    }
    const float v[16] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                         bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w),
                         bf16_lo(b.x), bf16_hi(b.x), bf16_lo(b.y), bf16_hi(b.y),
                         bf16_lo(b.z), bf16_hi(b.z), bf16_lo(b.w), bf16_hi(b.w)};
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    const float sc = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
    uint32_t packed[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t lo = ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i], sc), __fdiv_rn(v[4 * i + 1], sc));
      const uint16_t hi =
          ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i + 2], sc), __fdiv_rn(v[4 * i + 3], sc));
      packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    if (act) {
      const uint4 code = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      for (int j = 0; j <= k; ++j) {
        const int r = rows[j];
        if (r < 0) continue;
        *reinterpret_cast<uint4*>(q + (size_t)r * d + c0) = code;
        if ((threadIdx.x & 7) == 0) s[(size_t)r * (d / 128) + c0 / 128] = sc;
      }
    }
  }
}

// The hidden state of the batched GEMV path, fp32 [R][f], re-quantised per row and
// 128-block exactly as the activations: s = amax / 448 (IEEE divide; 1 if amax = 0),
// q = e4m3(h / s) rounded to nearest even.  8 threads per block, 16 values each.
__global__ void __launch_bounds__(256) quant_h_kernel(const float* __restrict__ h, int f,
                                                      uint8_t* __restrict__ q,
                                                      float* __restrict__ s) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // h comes from the gate/up kernel
  const float* hr = h + (size_t)blockIdx.x * f;
  const int lane16 = (threadIdx.x & 31) * 16;
  for (int c0 = threadIdx.x * 16; c0 - lane16 < f; c0 += blockDim.x * 16) {
    const bool act = c0 < f;
    float v[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 a = act ? __ldcg(reinterpret_cast<const float4*>(hr + c0) + i)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      v[4 * i] = a.x;
      v[4 * i + 1] = a.y;
      v[4 * i + 2] = a.z;
      v[4 * i + 3] = a.w;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    const float sc = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
    uint32_t packed[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t lo = ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i], sc), __fdiv_rn(v[4 * i + 1], sc));
      const uint16_t hi =
          ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i + 2], sc), __fdiv_rn(v[4 * i + 3], sc));
      packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    if (act) {
      *reinterpret_cast<uint4*>(q + (size_t)blockIdx.x * f + c0) =
          make_uint4(packed[0], packed[1], packed[2], packed[3]);
      if ((threadIdx.x & 7) == 0) s[(size_t)blockIdx.x * (f / 128) + c0 / 128] = sc;
    }
  }
}

}  // namespace

cudaError_t launch_quant_h(const float* h, int R, int f, uint8_t* q, float* s, cudaStream_t st,
                           bool overlap) {
  int threads = (f / 16 + 31) / 32 * 32;
  if (threads > 256) threads = 256;
  return launch_pdl(quant_h_kernel, dim3((unsigned)R), dim3(threads), 0, st, overlap, h, f, q, s);
}

cudaError_t launch_quant_rows(const uint16_t* x, int T, int k, int d, const int32_t* perm,
                              int nrows_routed, uint8_t* q, float* s, const int32_t* offsets,
                              int E, int nmax, int32_t* plan, int* counters, size_t n_counters,
                              int* status, cudaStream_t st, int plan_mode, bool overlap,
                              int32_t* ipos) {
  if (perm != nullptr && ipos != nullptr && nrows_routed == T * k && k <= 32 && plan_mode != 1 &&
      nrows_routed >= kQuantTokensMinPairs) {
    // each token quantised once: the inverse permutation, then one block per token
    const int P = T * k;
    const unsigned ib = (unsigned)((P + 255) / 256 < 4 * 148 ? (P + 255) / 256 : 4 * 148);
    cudaError_t e = launch_pdl(invperm_kernel, dim3(ib > 0 ? ib : 1), dim3(256), 0, st, overlap, perm,
                               P, ipos, status);
    if (e != cudaSuccess) return e;
    int threads = (d / 16 + 31) / 32 * 32;
    if (threads > 256) threads = 256;
    if (threads < 64) threads = 64;  // the row list takes up to k + 1 = 33 threads
    const unsigned blocks = (unsigned)(T + (plan != nullptr ? 1 : 0));
    return launch_pdl(quant_tokens_kernel, dim3(blocks), dim3(threads), 0, st, true, x, T, k, d,
                      ipos, q, s, offsets, E, nmax, plan, counters, n_counters, status, plan_mode);
  }
  const int R = nrows_routed + T;
  const unsigned blocks = (unsigned)(R + (plan != nullptr ? 1 : 0));
  int threads = (d / 16 + 31) / 32 * 32;  // whole warps
  if (threads > 256) threads = 256;
  return launch_pdl(quant_rows_kernel, dim3(blocks), dim3(threads), 0, st, overlap, x, T, k, d, perm,
                    nrows_routed, q, s, offsets, E, nmax, plan, counters, n_counters, status,
                    plan_mode);
}

}  // namespace bitmoe
