// Routing-weighted combine: out[t] = y_shared[t] + sum_{j<k} w[t,j] * y_routed[pos[t*k+j]],
// accumulated in fp32 in fixed j order (tcti.cn post, "DeepSeek-V4-Flash的可能性": the
// always-on shared expert is added beside the routed ones).  A row of CTAs per token,
// each taking a slice of the d outputs with 16-byte vector loads and stores.
#include "internal.cuh"
#include "ptx.cuh"

namespace bitmoe {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y,
                                                      const float* __restrict__ ysh,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ pos, int T,
                                                      int k, int d, float* __restrict__ out,
                                                      int* __restrict__ status) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // y, y_shared, w and pos come from earlier work on the stream
  __shared__ float sw[32];
  __shared__ int32_t sp[32];
  const int t = blockIdx.x;  // token; blockIdx.y: which slice of the row
  const int P = T * k;
  if (threadIdx.x < k) {
    int p = pos[(size_t)t * k + threadIdx.x];
    float wt = w[(size_t)t * k + threadIdx.x];
    if (p < 0 || p >= P) {  // not a valid row of y: flag and leave it out
      if (blockIdx.y == 0) atomicOr(status, kStatusBadIndex);
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
  for (int i = blockIdx.y * blockDim.x + threadIdx.x; i < nv; i += gridDim.y * blockDim.x) {
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

// Grid: one row of CTAs per token, each CTA one float4 per thread of a slice of the row
// (a short row needs one round of loads, whatever T is).
cudaError_t launch_combine(const float* y, const float* ysh, const float* w, const int32_t* pos,
                           int T, int k, int d, float* out, int* status, cudaStream_t s,
                           bool overlap) {
  int threads = d / 4 < 256 ? d / 4 : 256;
  threads = (threads + 31) / 32 * 32;
  const unsigned slices = (unsigned)((d / 4 + threads - 1) / threads);
  return launch_pdl(combine_kernel, dim3((unsigned)T, slices), dim3(threads), 0, s, overlap, y, ysh, w, pos,
                    T, k, d, out, status);
}

}  // namespace bitmoe
