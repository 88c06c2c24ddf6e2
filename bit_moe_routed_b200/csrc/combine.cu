// Routing-weighted combine: out[t] = y_shared[t] + sum_{j<k} w[t,j] * y_routed[pos[t*k+j]],
// accumulated in fp32 in fixed j order (tcti.cn post, "DeepSeek-V4-Flash的可能性": the
// always-on shared expert is added beside the routed ones).  One CTA per token,
// 16-byte vector loads and stores.
#include "internal.cuh"

namespace bitmoe {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y,
                                                      const float* __restrict__ ysh,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ pos, int T,
                                                      int k, int d, float* __restrict__ out,
                                                      int* __restrict__ status) {
  __shared__ float sw[32];
  __shared__ int32_t sp[32];
  const int t = blockIdx.x;
  const int P = T * k;
  if (threadIdx.x < k) {
    int p = pos[(size_t)t * k + threadIdx.x];
    float wt = w[(size_t)t * k + threadIdx.x];
    if (p < 0 || p >= P) {  // not a valid row of y: flag and leave it out
      atomicOr(status, kStatusBadIndex);
      p = -1;
      wt = 0.f;
    }
    sp[threadIdx.x] = p;
    sw[threadIdx.x] = wt;
  }
  __syncthreads();
  const int nv = d / 4;
  const float4* sh4 = reinterpret_cast<const float4*>(ysh + (size_t)t * d);
  float4* o4 = reinterpret_cast<float4*>(out + (size_t)t * d);
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    float4 acc = sh4[i];
    for (int j = 0; j < k; ++j) {
      if (sp[j] < 0) continue;
      const float4 v = reinterpret_cast<const float4*>(y + (size_t)sp[j] * d)[i];
      const float wj = sw[j];
      acc.x = fmaf(wj, v.x, acc.x);
      acc.y = fmaf(wj, v.y, acc.y);
      acc.z = fmaf(wj, v.z, acc.z);
      acc.w = fmaf(wj, v.w, acc.w);
    }
    o4[i] = acc;
  }
}

}  // namespace

cudaError_t launch_combine(const float* y, const float* ysh, const float* w, const int32_t* pos,
                           int T, int k, int d, float* out, int* status, cudaStream_t s) {
  int threads = d / 4 < 256 ? d / 4 : 256;
  threads = (threads + 31) / 32 * 32;
  combine_kernel<<<(unsigned)T, threads, 0, s>>>(y, ysh, w, pos, T, k, d, out, status);
  return cudaGetLastError();
}

}  // namespace bitmoe
