// moe_expert_ffn_noalloc: the expert FFN with its scratch memory in a fixed device array
// that the library itself owns, so the caller never has to allocate a workspace.
//
// Some callers cannot allocate device memory at the point where they run the layer: a
// plugin inside an inference engine that was given no workspace slot, or a serving loop
// that must not call cudaMalloc (it can synchronise the device and stall every stream).
// They pass only inputs and outputs here; the quantised rows, the hidden state and the
// tile plan live in `g_noalloc_scratch` below.
//
// Costs and rules of use:
//  - Every GPU that loads this library holds MOE_NOALLOC_SCRATCH_BYTES (24 MiB) for this
//    array until the process exits.
//  - Calls whose workspace would exceed that size are rejected with MOE_ERR_WORKSPACE.
//  - All calls share the one array per device.  Two calls that overlap on the GPU (on
//    different streams, or from different threads without ordering) race on it.
//  - The array keeps the last call's contents.  Nothing in it needs to start at zero:
//    each call writes the tile plan and every quantised row before reading them.
//  - The first call on each device looks up the array's device address
//    (cudaGetSymbolAddress, with that device current), checks the result and caches it.
#include "../../include/bitmoe.h"
#include "internal.cuh"

#include <atomic>
#include <cstdio>
#include <mutex>

namespace bitmoe {
namespace {

// Device-side scratch; in host code this name is only a stand-in, never a device address.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<int> g_ready[kMaxDevices];
uint8_t* g_addr[kMaxDevices];
std::mutex g_mu;

// Device address of the scratch array on the current device (looked up once per device).
int scratch_address(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "cudaGetDevice: %s", cudaGetErrorString(e));
    return record_error(MOE_ERR_CUDA, msg);
  }
  if (dev < 0 || dev >= kMaxDevices) return record_error(MOE_ERR_UNSUPPORTED, "device index");
  if (!g_ready[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ready[dev].load(std::memory_order_relaxed)) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr) {
        char msg[256];
        snprintf(msg, sizeof(msg), "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        return record_error(MOE_ERR_CUDA, msg);
      }
      g_addr[dev] = static_cast<uint8_t*>(p);
      g_ready[dev].store(1, std::memory_order_release);
    }
  }
  *out = g_addr[dev];
  return MOE_OK;
}

}  // namespace
}  // namespace bitmoe

extern "C" int moe_expert_ffn_noalloc(const uint16_t* x_bf16, int T, int k,
                                      const moe_weights_t* w, const int32_t* offsets,
                                      const int32_t* perm, float* y_routed, float* y_shared,
                                      void* stream) {
  using namespace bitmoe;
  if (w == nullptr) return record_error(MOE_ERR_INVALID_ARG, "weights descriptor is NULL");
  const size_t need = moe_workspace_size(T, k, w->E, w->d, w->f);
  if (need == 0)
    return record_error(MOE_ERR_INVALID_ARG, "invalid sizes (T, k, E, d or f)");
  if (need > (size_t)MOE_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "T=%d k=%d E=%d d=%d f=%d needs %zu bytes of scratch, more than the fixed %u; "
             "use moe_expert_ffn with a caller-owned workspace",
             T, k, w->E, w->d, w->f, need, (unsigned)MOE_NOALLOC_SCRATCH_BYTES);
    return record_error(MOE_ERR_WORKSPACE, msg);
  }
  if (T == 0) return MOE_OK;
  uint8_t* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc) return rc;
  return moe_expert_ffn(x_bf16, T, k, w, offsets, perm, y_routed, y_shared, scratch,
                        (size_t)MOE_NOALLOC_SCRATCH_BYTES, stream);
}
