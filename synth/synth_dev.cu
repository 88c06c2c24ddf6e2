// Seeded synthetic FP4 expert weights, device side.
//
// Input generator only: it holds none of the MoE method's arithmetic.  It
// writes the same bytes as synth_host.c (SplitMix64, Steele/Lea/Flood 2014,
// Vigna's constants), implemented here again from the generator's published
// definition so that a layer's weights (13.4 MB per expert at d=4096, f=2048,
// 147.7 GB for 43 layers) can be made where they live, in HBM.
//
// Stream id = ((layer * 1024 + expert) * 4 + matrix) * 2 + kind; initial state
// s0 = seed ^ (id << 40); byte i of a matrix = byte (i % 8) of output
// floor(i / 8) + 1; codes use the byte as is, scales use 121 + (byte & 3).
#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t splitmix_output(uint64_t s0, uint64_t n) {
  uint64_t z = s0 + n * 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// One thread per 8-byte word of each expert's matrix; experts are contiguous
// blocks of `bytes_per_expert` bytes starting at `out`.
__global__ void fill_kernel(uint64_t seed, int layer, int n_experts, int matrix, int kind,
                            size_t bytes_per_expert, uint8_t* __restrict__ out) {
  const size_t words_per_expert = (bytes_per_expert + 7) / 8;
  const size_t total = words_per_expert * (size_t)n_experts;
  for (size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(g / words_per_expert);
    const size_t w = g - (size_t)e * words_per_expert;
    const uint64_t sid = ((((uint64_t)layer * 1024u + (uint64_t)e) * 4u + (uint64_t)matrix) * 2u +
                          (uint64_t)kind);
    const uint64_t word = splitmix_output(seed ^ (sid << 40), (uint64_t)w + 1u);
    uint8_t* dst = out + (size_t)e * bytes_per_expert + w * 8;
    const size_t left = bytes_per_expert - w * 8;
    if (kind == 0 && left >= 8 && (((uintptr_t)dst) & 7u) == 0) {
      *reinterpret_cast<uint64_t*>(dst) = word;
    } else {
      for (unsigned k = 0; k < 8u && k < left; ++k) {
        uint8_t v = (uint8_t)(word >> (8u * k));
        dst[k] = kind == 0 ? v : (uint8_t)(121u + (v & 3u));
      }
    }
  }
}

}  // namespace

extern "C" int synth_fill_dev(uint64_t seed, int layer, int n_experts, int matrix, int kind,
                              size_t bytes_per_expert, void* out, void* stream) {
  if (out == nullptr || n_experts <= 0 || bytes_per_expert == 0) return -1;
  const size_t words = (bytes_per_expert + 7) / 8 * (size_t)n_experts;
  size_t blocks = (words + 255) / 256;
  if (blocks > 148u * 64u) blocks = 148u * 64u;
  fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      seed, layer, n_experts, matrix, kind, bytes_per_expert, (uint8_t*)out);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
