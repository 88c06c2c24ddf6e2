// FP8 x FP8 GEMM for a few tokens, and the FP8-weight shared expert built on it.
//
// The pages' software stack has an fp8_gemm beside fp4_gemm (tcti.cn post, "补齐软件栈缺失":
// FP8 activations times FP8 weights, the format of the model's linears that are not FP4);
// the shared expert of the real model is one of them.  The page gives no scale layout;
// this library reads it as e4m3 weights with one fp32 scale per 128 x 128 block (rows x
// reduction) and activations quantised per token and 128-element block to e4m3 with
// scale amax / 448, as for the FP4 path:
//   C[m][n] = sum_kb sa[m][kb] sb[n/128][kb] sum_{k in kb} A[m][k] B[n][k].
//
// For M <= 64 tokens the product is bound by reading B once.  Work is cut into tasks of
// 16 weight rows x 512 reduction elements; a CTA of four warps takes four tasks of the
// same 512-element chunk, one per warp.  The CTA copies the chunk of every token's row
// (M x 512 bytes) and each warp its task's 16 weight rows (8 KB) into shared memory with
// 16-byte cp.async, rows padded to 544 bytes so that the eight rows one 8-byte read
// touches fall on different banks.  Per 32-element block the warp then runs one
// mma.sync m16n8k32 e4m3 per group of 8 tokens straight on the codes (no decode): lane
// (g, t) holds bytes 8t..8t+7 of the block in rows g and g+8 (k-slots 4t..4t+3 and
// 16+4t..16+4t+3) and the same 8 bytes of token g's row.  Four blocks (128 elements) sum
// in the tensor core; then the block's weight scale and the token's scale are applied in
// fp32.  Each task leaves its partial sums in the workspace, and the last of a row
// block's tasks to finish (an acq_rel counter) adds them in reduction order and writes
// the result, so results do not depend on timing.  With two weight matrices (the gate and
// up projections of one expert) the 16 rows are 8 gate and the same 8 up rows and the
// result is h = silu(g) * u.
#include "internal.cuh"
#include "ptx.cuh"

namespace bitmoe {
namespace {

constexpr int kF8Warps = 4;                 // warps per CTA, one task each
constexpr int kF8Rows = 16;                 // weight rows per task (the MMA's M)
constexpr int kF8K = 512;                   // reduction elements per task
constexpr int kF8Pitch = kF8K + 32;         // shared-memory row pitch in bytes

struct Fp8Params {
  const uint8_t* A;    // activations [M][K] e4m3
  const float* sa;     // [M][K/128]
  const uint8_t* B0;   // weights [N][K] e4m3
  const float* sb0;    // [N/128][K/128]
  const uint8_t* B1;   // second weight matrix (fused gate/up) or null
  const float* sb1;
  int M, N, K;
  float* part;         // [units][K/512][16 rows][M8] partial sums
  int* cnt;            // [units] arrivals; zero on entry, the last arrival zeroes it again
  float* C;            // [M][N]
};

__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

// shared memory of a CTA: four weight tiles, then the tokens' rows of the chunk
__host__ __device__ constexpr int fp8_smem_bytes(int M) {
  return kF8Warps * kF8Rows * kF8Pitch + ((M + 7) / 8 * 8) * kF8Pitch;
}

template <int NS, bool FUSED>
__global__ void __launch_bounds__(kF8Warps * 32) fp8_gemm_kernel(const Fp8Params p) {
  extern __shared__ __align__(16) uint8_t f8_smem[];
  ptx::griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int K = p.K, M = p.M, kc = K / kF8K, nkb = K / 128;
  const int M8 = NS * 8;
  const int units = FUSED ? p.N / 8 : p.N / 16;  // a multiple of kF8Warps (N % 128 == 0)
  const int per_chunk = units / kF8Warps;
  const int chunk = blockIdx.x / per_chunk;
  const int unit = (blockIdx.x % per_chunk) * kF8Warps + warp;
  const int row0 = FUSED ? 8 * unit : 16 * unit;  // first weight row (of each matrix)
  uint8_t* wt = f8_smem + warp * kF8Rows * kF8Pitch;
  uint8_t* at = f8_smem + kF8Warps * kF8Rows * kF8Pitch;

  // this warp's 16 weight rows (they do not depend on earlier work: copied while the
  // previous kernel on the stream may still run), then the CTA's tokens (M rows x 512
  // bytes of the chunk)
  for (int i = lane; i < kF8Rows * (kF8K / 16); i += 32) {
    const int r = i / (kF8K / 16), c16 = i % (kF8K / 16);
    const uint8_t* src = FUSED ? (r < 8 ? p.B0 + (size_t)(row0 + r) * K
                                        : p.B1 + (size_t)(row0 + r - 8) * K)
                               : p.B0 + (size_t)(row0 + r) * K;
    ptx::cp_async_16(ptx::smem_u32(wt + r * kF8Pitch + 16 * c16), src + chunk * kF8K + 16 * c16);
  }
  ptx::griddep_wait();  // A, its scales and the counters come from earlier work
  for (int i = threadIdx.x; i < M * (kF8K / 16); i += kF8Warps * 32) {
    const int r = i / (kF8K / 16), c16 = i % (kF8K / 16);
    ptx::cp_async_16(ptx::smem_u32(at + r * kF8Pitch + 16 * c16),
                     p.A + (size_t)r * K + chunk * kF8K + 16 * c16);
  }
  ptx::cp_async_commit();
  ptx::cp_async_wait_all();
  __syncthreads();  // every thread's copies of the tokens have landed

  // rows g and g+8 of the task; tokens 8s + 2t, 8s + 2t + 1 of group s
  float acc[NS][4];
#pragma unroll
  for (int s = 0; s < NS; ++s)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[s][i] = 0.f;
  const int rowblk = row0 / 128;
#pragma unroll
  for (int sc = 0; sc < kF8K / 128; ++sc) {
    const int kb = chunk * (kF8K / 128) + sc;  // the 128-block of the reduction
    float cq[NS][4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int kk = sc * 128 + b * 32 + 8 * t;  // lane's 8 bytes of the 32-block
      const uint2 wa = *reinterpret_cast<const uint2*>(wt + g * kF8Pitch + kk);
      const uint2 wb = *reinterpret_cast<const uint2*>(wt + (g + 8) * kF8Pitch + kk);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        const int tok = 8 * s + g;
        uint2 xv = make_uint2(0u, 0u);
        if (tok < M) xv = *reinterpret_cast<const uint2*>(at + tok * kF8Pitch + kk);
        if (b == 0)
          ptx::mma_m16n8k32_e4m3_zero(cq[s], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
        else
          ptx::mma_m16n8k32_e4m3(cq[s], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
      }
    }
    const float sba = __ldg(p.sb0 + (size_t)rowblk * nkb + kb);
    const float sbb = FUSED ? __ldg(p.sb1 + (size_t)rowblk * nkb + kb) : sba;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int t0 = 8 * s + 2 * t, t1 = t0 + 1;
      const float s0 = t0 < M ? __ldg(p.sa + (size_t)t0 * nkb + kb) : 0.f;
      const float s1 = t1 < M ? __ldg(p.sa + (size_t)t1 * nkb + kb) : 0.f;
      acc[s][0] = fmaf(s0, sba * cq[s][0], acc[s][0]);
      acc[s][1] = fmaf(s1, sba * cq[s][1], acc[s][1]);
      acc[s][2] = fmaf(s0, sbb * cq[s][2], acc[s][2]);
      acc[s][3] = fmaf(s1, sbb * cq[s][3], acc[s][3]);
    }
  }

  // partials of (row, token): rows g and g+8, tokens 8s + 2t + {0, 1}
  float* pp = p.part + (size_t)(unit * kc + chunk) * kF8Rows * M8;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const int t0 = 8 * s + 2 * t;
    *reinterpret_cast<float2*>(pp + g * M8 + t0) = make_float2(acc[s][0], acc[s][1]);
    *reinterpret_cast<float2*>(pp + (g + 8) * M8 + t0) = make_float2(acc[s][2], acc[s][3]);
  }
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atom_add_acq_rel(p.cnt + unit, 1) == kc - 1 ? 1 : 0;
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __syncwarp();  // lane 0's acquire orders the whole warp's loads below
  // the last task of the row block: sum the partials in reduction order
  const float* base = p.part + (size_t)unit * kc * kF8Rows * M8;
  if (FUSED) {
    for (int i = lane; i < 8 * M; i += 32) {
      const int r = i / M, tok = i % M;
      float gg = 0.f, uu = 0.f;
      for (int c = 0; c < kc; ++c) {
        gg += __ldcg(base + ((size_t)c * kF8Rows + r) * M8 + tok);
        uu += __ldcg(base + ((size_t)c * kF8Rows + r + 8) * M8 + tok);
      }
      p.C[(size_t)tok * p.N + row0 + r] = __fdividef(gg, 1.0f + expf(-gg)) * uu;
    }
  } else {
    for (int i = lane; i < kF8Rows * M; i += 32) {
      const int r = i / M, tok = i % M;
      float y = 0.f;
      for (int c = 0; c < kc; ++c) y += __ldcg(base + ((size_t)c * kF8Rows + r) * M8 + tok);
      p.C[(size_t)tok * p.N + row0 + r] = y;
    }
  }
  if (lane == 0) p.cnt[unit] = 0;  // ready for the next launch on the stream
}

template <int NS, bool FUSED>
cudaError_t launch_kern(const Fp8Params& prm, cudaStream_t s, bool overlap) {
  const int units = FUSED ? prm.N / 8 : prm.N / 16;
  const int ctas = units / kF8Warps * (prm.K / kF8K);
  const size_t smem = (size_t)fp8_smem_bytes(prm.M);
  auto kern = fp8_gemm_kernel<NS, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)ctas), dim3(kF8Warps * 32), smem, s, overlap, prm);
}

template <bool FUSED>
cudaError_t launch_ns(const Fp8Params& prm, int ns, cudaStream_t s, bool overlap) {
  switch (ns) {
    case 1: return launch_kern<1, FUSED>(prm, s, overlap);
    case 2: return launch_kern<2, FUSED>(prm, s, overlap);
    case 4: return launch_kern<4, FUSED>(prm, s, overlap);
    default: return launch_kern<8, FUSED>(prm, s, overlap);
  }
}

int groups_for(int M) {
  const int n = (M + 7) / 8;
  return n <= 1 ? 1 : n <= 2 ? 2 : n <= 4 ? 4 : 8;
}

size_t part_bytes(int M, int N, int K, bool fused) {
  const int units = fused ? N / 8 : N / 16;
  return (size_t)units * (K / kF8K) * kF8Rows * (groups_for(M) * 8) * sizeof(float);
}

}  // namespace

size_t fp8_gemm_ws_bytes(int M, int N, int K, bool fused) {
  const int units = fused ? N / 8 : N / 16;
  return (part_bytes(M, N, K, fused) + 255) / 256 * 256 + (size_t)units * sizeof(int);
}

size_t fp8_gemm_counters(int N, bool fused) { return (size_t)(fused ? N / 8 : N / 16); }

cudaError_t launch_fp8_gemm(const Fp8Launch& a, cudaStream_t s) {
  Fp8Params p;
  p.A = a.A;
  p.sa = a.sa;
  p.B0 = a.B0;
  p.sb0 = a.sb0;
  p.B1 = a.B1;
  p.sb1 = a.sb1;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  const bool fused = a.B1 != nullptr;
  p.part = reinterpret_cast<float*>(a.ws);
  p.cnt = a.cnt ? a.cnt
                : reinterpret_cast<int*>(a.ws + (part_bytes(a.M, a.N, a.K, fused) + 255) / 256 * 256);
  p.C = a.C;
  if (a.zero_counters) {
    cudaError_t e = cudaMemsetAsync(p.cnt, 0, fp8_gemm_counters(a.N, fused) * sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  const int ns = groups_for(a.M);
  return fused ? launch_ns<true>(p, ns, s, a.overlap) : launch_ns<false>(p, ns, s, a.overlap);
}

}  // namespace bitmoe
