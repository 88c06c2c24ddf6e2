// C ABI of libbitmoe.so: argument checks, workspace layout, error reporting, and the
// launches of the routing, dispatch, quantisation, expert-FFN and combine kernels.
// The calls follow the pages' statement of the problem: route (dpshk.com article,
// "核心实现一"), group tokens per expert (same article, "核心实现三"), fused low-bit FFN
// (same article, "核心实现四"; tcti.cn post, "补齐软件栈缺失"), weighted combine.
#include "../../include/bitmoe.h"
#include "internal.cuh"

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

namespace bitmoe {

__device__ int g_status;  // device status word (kStatus* bits), one per device

namespace {

thread_local std::string t_err;
// Set while a call issues kernels that follow another of this library's kernels on the
// stream (see launch_pdl): they may start while it finishes.
thread_local bool t_overlap = false;
struct OverlapScope {
  bool saved;
  OverlapScope() : saved(t_overlap) { t_overlap = true; }
  ~OverlapScope() { t_overlap = saved; }
};
std::atomic<long long> g_wait_ns{2000000000LL};
std::atomic<int> g_gemv_max_t{kBgMaxT};  // batches up to this size take a GEMV path
std::atomic<int> g_stall{0};                 // test knob: see moe_set_test_stall
std::atomic<int> g_decode_engine{0};         // see moe_set_decode_engine

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct DeviceInfo {
  int sms = 0;
  int status_ok = 0;
  int* status = nullptr;
};

// Per-device facts, looked up once per device (SM count, sm_100 check, status address).
int device_info(DeviceInfo& out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  static DeviceInfo cache[64];
  static std::atomic<int> ready[64];
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
  if (ready[dev].load(std::memory_order_acquire)) {
    out = cache[dev];
    return MOE_OK;
  }
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(MOE_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                prop.major, prop.minor);
  DeviceInfo d;
  d.sms = prop.multiProcessorCount;
  void* sp = nullptr;
  e = cudaGetSymbolAddress(&sp, g_status);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
  d.status = static_cast<int*>(sp);
  cache[dev] = d;
  ready[dev].store(1, std::memory_order_release);
  out = d;
  return MOE_OK;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int check_weights(const moe_weights_t* w) {
  if (w == nullptr) return fail(MOE_ERR_INVALID_ARG, "weights descriptor is NULL");
  if (!w->gate_codes || !w->gate_scales || !w->up_codes || !w->up_scales || !w->down_codes ||
      !w->down_scales)
    return fail(MOE_ERR_INVALID_ARG, "a weight pointer is NULL");
  if (w->E < 1 || w->E > 1024) return fail(MOE_ERR_INVALID_ARG, "E=%d outside [1, 1024]", w->E);
  if (w->d < 128 || w->d % 128 || w->f < 128 || w->f % 128)
    return fail(MOE_ERR_INVALID_ARG, "d=%d, f=%d must be positive multiples of 128", w->d, w->f);
  if (w->d > 8192 || w->f > 8192)
    return fail(MOE_ERR_INVALID_ARG, "d=%d, f=%d: at most 8192 supported", w->d, w->f);
  if (!aligned(w->gate_codes, 32) || !aligned(w->up_codes, 32) || !aligned(w->down_codes, 32))
    return fail(MOE_ERR_INVALID_ARG, "weight code arrays must be 32-byte aligned");
  if (!aligned(w->gate_scales, 4) || !aligned(w->up_scales, 4) || !aligned(w->down_scales, 4))
    return fail(MOE_ERR_INVALID_ARG, "weight scale arrays must be 4-byte aligned");
  return MOE_OK;
}

}  // namespace

EncodeTiledFn tensor_map_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D map over a byte matrix [rows][cols]; box = box_cols bytes x box_rows rows, no swizzle.
bool make_byte_map(CUtensorMap* m, const void* base, long long cols, long long rows, int box_cols,
                   int box_rows) {
  EncodeTiledFn fn = tensor_map_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over byte rows [rows][cols] viewed as (128-byte piece, row, piece index): a box of
// `pieces` pieces x box_rows rows lands as [piece][row][128 bytes] with the 128-byte swizzle
// (16-byte chunk index XOR row mod 8).  Rows past the end read as zeros.
bool make_code_map(CUtensorMap* m, const void* base, long long cols, long long rows, int box_rows,
                   int pieces) {
  EncodeTiledFn fn = tensor_map_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {128u, (cuuint64_t)rows, (cuuint64_t)(cols / 128)};
  const cuuint64_t strides[2] = {(cuuint64_t)cols, 128u};
  const cuuint32_t box[3] = {128u, (cuuint32_t)box_rows, (cuuint32_t)pieces};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over an fp32 matrix [rows][cols]; box = cols x box_rows (cols*4 a multiple of 16).
bool make_f32_map(CUtensorMap* m, const void* base, long long cols, long long rows, int box_rows) {
  EncodeTiledFn fn = tensor_map_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  const cuuint32_t box[2] = {(cuuint32_t)cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Sets the message moe_last_error returns, for the library's other translation units.
int record_error(int code, const char* msg) { return fail(code, "%s", msg); }

WorkspaceLayout workspace_layout(int T, int k, int E, int d, int f) {
  WorkspaceLayout L{};
  const size_t R = (size_t)T * k + T;
  size_t o = 0;
  L.plan = o;
  // the tile plan, or (batched GEMV) the slot count and (expert, row, rows) per slot
  size_t plan_ints = (size_t)E + 2 + 2 * plan_ntmax((int)R, E);
  if (T <= kBgMaxT && 1 + 3 * R > plan_ints) plan_ints = 1 + 3 * R;
  o = align256(o + 4 * plan_ints);
  L.qx = o;
  o = align256(o + R * d);
  L.sx = o;
  o = align256(o + R * (d / 128) * 4);
  L.qh = o;
  o = align256(o + R * f);
  L.sh = o;
  o = align256(o + R * (f / 128) * 4);
  L.counters = o;
  const size_t hb = (size_t)((d > f ? d : f) / 128);
  L.n_counters = plan_ntmax((int)R, E) * hb;
  o = align256(o + 4 * L.n_counters);
  // stream-K partial slots of the tile kernels: two per CTA, each [ncap columns][2 matrices]
  // [tile rows] fp32 (small batches take tiles of up to 256 weight rows, large ones 128).
  // The GEMV paths' fp32 hidden state (single token: per active expert; batched: per row)
  // shares the area: a call runs either the tile kernels or a GEMV path, never both.
  L.partials = o;
  L.hbuf = o;
  const size_t tile_rows_max = nmax_for(T) == kNmaxSmall ? 256 : 128;
  size_t area = (size_t)kMaxCtas * 2 * (size_t)ncap_for(T) * 2 * tile_rows_max * 4;
  if (T <= kBgMaxT && R * f * 4 > area) area = R * f * 4;
  o = align256(o + area);
  // the combine counters of the single-token kernel (one per 16 output rows)
  L.done2 = o;
  if (T <= kGemvMaxT) o = align256(o + 4 * (size_t)(d / 16));
  // the pieces and counters of the tensor-core single-token kernel
  L.dtc = o;
  if (T <= kGemvMaxT) o = align256(o + decode_tc_ws_bytes(k, d, f));
  // the multi-CTA dispatch's counts (moe_forward on large batches)
  L.dispatch = o;
  o = align256(o + dispatch_ws_bytes(T, k, E));
  // the inverse of the dispatch permutation (the prepare step's row of each pair)
  L.ipos = o;
  o = align256(o + 4 * (size_t)T * k);
  L.total = o;
  return L;
}

}  // namespace bitmoe

using namespace bitmoe;

extern "C" {

const char* moe_last_error(void) { return t_err.c_str(); }

int moe_set_wait_limit_ns(long long n) {
  g_wait_ns.store(n > 0 ? n : 2000000000LL);
  return MOE_OK;
}

int moe_set_test_stall(int on) {
  g_stall.store(on ? 1 : 0);
  return MOE_OK;
}

int moe_set_decode_engine(int engine) {
  if (engine != 0 && engine != 1) return fail(MOE_ERR_INVALID_ARG, "engine=%d is not 0 or 1", engine);
  g_decode_engine.store(engine);
  return MOE_OK;
}

int moe_set_gemv_max_tokens(int t) {
  if (t < 0) return fail(MOE_ERR_INVALID_ARG, "t=%d < 0", t);
  g_gemv_max_t.store(t);
  return MOE_OK;
}

size_t moe_dispatch_workspace_size(int T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  return dispatch_ws_bytes(T, k, E);
}

size_t moe_workspace_size(int T, int k, int E, int d, int f) {
  if (T < 0 || k < 1 || E < 1 || d < 128 || f < 128 || d % 128 || f % 128) return 0;
  return workspace_layout(T, k, E, d, f).total;
}

int moe_workspace_offsets(int T, int k, int E, int d, int f, size_t off[5]) {
  if (off == nullptr) return fail(MOE_ERR_INVALID_ARG, "off is NULL");
  if (moe_workspace_size(T, k, E, d, f) == 0)
    return fail(MOE_ERR_INVALID_ARG, "invalid sizes T=%d k=%d E=%d d=%d f=%d", T, k, E, d, f);
  const WorkspaceLayout L = workspace_layout(T, k, E, d, f);
  off[0] = L.qx;
  off[1] = L.sx;
  off[2] = L.qh;
  off[3] = L.sh;
  off[4] = T <= kBgMaxT ? L.hbuf : (size_t)-1;
  return MOE_OK;
}

int moe_sync_status(void* stream) {
  DeviceInfo di;
  int rc = device_info(di);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int host = 0;
  e = cudaMemcpy(&host, di.status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  if (host != 0) {
    const int zero = 0;
    e = cudaMemcpy(di.status, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear status");
    if (host & kStatusTimeout) {
      // a CTA that gave up may have left the single-token kernel's grid barrier mid-count
      e = reset_grid_barrier();
      if (e == cudaSuccess) e = reset_tc_barrier(di.sms < kMaxCtas ? di.sms : kMaxCtas);
      if (e != cudaSuccess) return cuda_fail(e, "reset grid barrier");
      return fail(MOE_ERR_TIMEOUT, "a device-side wait exceeded its limit (status 0x%x)", host);
    }
    return fail(MOE_ERR_INVALID_ARG, "an expert id or position was out of range (status 0x%x)",
                host);
  }
  return MOE_OK;
}

int moe_route_topk(const float* scores, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                   void* stream) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  if (E < 1 || E > 1024) return fail(MOE_ERR_INVALID_ARG, "E=%d outside [1, 1024]", E);
  if (k < 1 || k > E || k > 32) return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, min(E, 32)]", k);
  if (T == 0) return MOE_OK;
  if (!scores || !topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(scores, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
    return fail(MOE_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  DeviceInfo di;
  int rc = device_info(di);
  if (rc) return rc;
  cudaError_t e =
      launch_route_topk(scores, T, E, k, topk_idx, topk_w, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "route_topk launch");
}

int moe_router_topk(const uint16_t* x_bf16, const uint16_t* w_router_bf16, int T, int d, int E,
                    int k, float* scores, int32_t* topk_idx, float* topk_w, void* stream) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  if (E < 1 || E > 1024) return fail(MOE_ERR_INVALID_ARG, "E=%d outside [1, 1024]", E);
  if (k < 1 || k > E || k > 32) return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, min(E, 32)]", k);
  if (d < 128 || d % 128) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 128", d);
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !w_router_bf16 || !scores || !topk_idx || !topk_w)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(x_bf16, 4) || !aligned(w_router_bf16, 4) || !aligned(scores, 4) ||
      !aligned(topk_idx, 4) || !aligned(topk_w, 4))
    return fail(MOE_ERR_INVALID_ARG, "pointers must be 4-byte aligned");
  DeviceInfo di;
  int rc = device_info(di);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_router(x_bf16, w_router_bf16, T, d, E, scores, s, t_overlap);
  if (e != cudaSuccess) return cuda_fail(e, "router launch");
  e = launch_route_topk(scores, T, E, k, topk_idx, topk_w, s, true);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "route_topk launch");
}

int moe_dispatch(const int32_t* topk_idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
                 int32_t* perm, int32_t* pos, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  if (E < 1 || E > 1024) return fail(MOE_ERR_INVALID_ARG, "E=%d outside [1, 1024]", E);
  if (k < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, E]", k);
  if ((long long)T * k > (1LL << 30)) return fail(MOE_ERR_INVALID_ARG, "T*k too large");
  if (!counts || !offsets) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (T > 0 && (!topk_idx || !perm || !pos)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  DeviceInfo di;
  int rc = device_info(di);
  if (rc) return rc;
  const size_t need = dispatch_ws_bytes(T, k, E);
  if (need > 0 && ws != nullptr && ws_bytes >= need && aligned(ws, 4)) {
    cudaError_t e = launch_dispatch_multi(topk_idx, T, k, E, counts, offsets, perm, pos,
                                          static_cast<int32_t*>(ws), di.status,
                                          static_cast<cudaStream_t>(stream), t_overlap);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "dispatch launch");
  }
  // T == 0 still writes counts = 0 and offsets = 0 (the kernel handles P == 0)
  cudaError_t e = launch_dispatch(topk_idx, T, k, E, counts, offsets, perm, pos, di.status,
                                  static_cast<cudaStream_t>(stream), t_overlap);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "dispatch launch");
}

int moe_act_quant(const uint16_t* x_bf16, int T, int d, uint8_t* qx, float* sx, void* stream) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  if (d < 128 || d % 128 || d > 16384)
    return fail(MOE_ERR_INVALID_ARG, "d=%d must be a multiple of 128 in [128, 16384]", d);
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !qx || !sx) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(x_bf16, 16) || !aligned(qx, 16) || !aligned(sx, 4))
    return fail(MOE_ERR_INVALID_ARG, "x and qx must be 16-byte aligned, sx 4-byte aligned");
  DeviceInfo di;
  int rc = device_info(di);
  if (rc) return rc;
  cudaError_t e = launch_quant_rows(x_bf16, T, 1, d, nullptr, 0, qx, sx, nullptr, 0, 0, nullptr,
                                    nullptr, 0, di.status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "act_quant launch");
}

namespace {

struct FfnCtx {
  DeviceInfo di;
  WorkspaceLayout L;
  int nmax;
  bool bg;     // batched GEMV path (bgemv.cu) instead of the tcgen05 tiles (ffn.cu)
  bool gemv;   // single-token GEMV path (gemv.cu) instead of the tcgen05 tiles (ffn.cu)
  bool fused;  // ... in one cooperative kernel (decode.cu), for the whole-call entry points
  bool tc;     // ... whose forward form runs on the tensor cores (decode_tc.cu)
  uint8_t* ws;
};

// The GEMV path needs whole 512-element stages along d and f, 16-byte aligned scale
// rows for its TMA boxes, every CTA's range of units within two experts and the
// kernel's unit bound, and its shared memory.
bool use_gemv(int T, int k, const moe_weights_t* w, int sms, int max_smem) {
  if (T < 1 || T > g_gemv_max_t.load() || T > kGemvMaxT) return false;
  if (w->d % 512 || w->f % 512) return false;
  if (!aligned(w->gate_scales, 16) || !aligned(w->up_scales, 16) || !aligned(w->down_scales, 16))
    return false;
  const long long ctas = sms < kMaxCtas ? sms : kMaxCtas;
  const long long experts = (long long)T * k + 1;  // at most this many active
  if (experts > ctas) return false;
  const long long units1 = experts * (w->f / 8), units2 = experts * (w->d / 16);
  const long long cap = (long long)gemv_max_units_per_cta() * ctas;
  if (units1 > cap || units2 > cap) return false;
  return gemv_smem_bytes(1, w->d) <= (size_t)max_smem &&
         gemv_smem_bytes(2, w->f) <= (size_t)max_smem;
}

int ffn_check(int T, int k, const moe_weights_t* w, void* ws, size_t ws_bytes, FfnCtx& c) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  int rc = check_weights(w);
  if (rc) return rc;
  if (k < 1 || k > w->E) return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, E]", k);
  if ((long long)T * (k + 1) > (1LL << 28)) return fail(MOE_ERR_INVALID_ARG, "T too large");
  rc = device_info(c.di);
  if (rc) return rc;
  c.L = workspace_layout(T, k, w->E, w->d, w->f);
  if (T > 0 && ws_bytes != (size_t)-1) {
    if (ws == nullptr || !aligned(ws, 256))
      return fail(MOE_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
    if (ws_bytes < c.L.total)
      return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, c.L.total);
  }
  c.nmax = nmax_for(T);
  c.ws = static_cast<uint8_t*>(ws);
  int max_smem = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const size_t need1 = ffn_smem_bytes(1, c.nmax, w->E, w->f);
  const size_t need2 = ffn_smem_bytes(2, c.nmax, w->E, w->d);
  const size_t need = need1 > need2 ? need1 : need2;
  if (need > (size_t)max_smem)
    return fail(MOE_ERR_INVALID_ARG, "shape needs %zu bytes of shared memory (> %d)", need,
                max_smem);
  c.gemv = use_gemv(T, k, w, c.di.sms, max_smem);
  c.bg = T >= 2 && T <= g_gemv_max_t.load() && T <= kBgMaxT && w->d % 512 == 0 &&
         w->f % 512 == 0 && aligned(w->gate_scales, 16) && aligned(w->up_scales, 16) &&
         aligned(w->down_scales, 16) && bgemv_smem_bytes(w->d) <= (size_t)max_smem &&
         bgemv_smem_bytes(w->f) <= (size_t)max_smem;
  const int ctas = c.di.sms < kMaxCtas ? c.di.sms : kMaxCtas;
  c.fused = c.gemv && decode_fits(k, w->d, w->f, ctas) &&
            decode_smem_bytes(w->d, w->f) <= (size_t)max_smem;
  c.tc = c.fused && g_decode_engine.load() == 1 && decode_tc_fits(k, w->d, w->f, ctas) &&
         decode_tc_smem_bytes(w->d, w->f) <= (size_t)max_smem;
  return MOE_OK;
}

BgLaunch bg_args(int T, int k, const moe_weights_t* w, const FfnCtx& c) {
  BgLaunch a{};
  a.plan = reinterpret_cast<const int32_t*>(c.ws + c.L.plan);
  a.hbuf = reinterpret_cast<float*>(c.ws + c.L.hbuf);
  a.E = w->E;
  a.d = w->d;
  a.f = w->f;
  a.P = T * k;
  a.R = T * k + T;
  a.wait_ns = g_wait_ns.load();
  a.status = c.di.status;
  a.overlap = t_overlap;
  return a;
}

GemvLaunch gemv_args(int T, int k, const moe_weights_t* w, const FfnCtx& c) {
  GemvLaunch a{};
  a.plan = reinterpret_cast<const int32_t*>(c.ws + c.L.plan);
  a.qx = c.ws + c.L.qx;
  a.sx = reinterpret_cast<const float*>(c.ws + c.L.sx);
  a.hbuf = reinterpret_cast<float*>(c.ws + c.L.hbuf);
  a.qh = c.ws + c.L.qh;
  a.sh = reinterpret_cast<float*>(c.ws + c.L.sh);
  a.E = w->E;
  a.d = w->d;
  a.f = w->f;
  a.P = T * k;
  a.wait_ns = g_wait_ns.load();
  a.status = c.di.status;
  a.stall = g_stall.load();
  a.overlap = t_overlap;
  return a;
}

FfnArgs ffn_args(int phase, int T, int k, const moe_weights_t* w, const FfnCtx& c) {
  FfnArgs a{};
  const int P = T * k;
  a.E = w->E;
  a.R = P + T;
  a.P = P;
  a.f = w->f;
  a.d = w->d;
  a.plan = reinterpret_cast<const int32_t*>(c.ws + c.L.plan);
  a.wait_ns = g_wait_ns.load();
  a.status = c.di.status;
  a.counters = reinterpret_cast<int*>(c.ws + c.L.counters);
  a.partials = reinterpret_cast<float*>(c.ws + c.L.partials);
  a.ncap = ncap_for(T);
  a.l2_hints = 1;  // weight boxes evict-first
  a.overlap = t_overlap;
  if (phase == 1) {
    a.a0_codes = w->gate_codes;
    a.a0_scales = w->gate_scales;
    a.a1_codes = w->up_codes;
    a.a1_scales = w->up_scales;
    a.b_codes = c.ws + c.L.qx;
    a.b_scales = reinterpret_cast<const float*>(c.ws + c.L.sx);
    a.K = w->d;
    a.rows_per_expert = w->f;
    a.qh = c.ws + c.L.qh;
    a.sh = reinterpret_cast<float*>(c.ws + c.L.sh);
  } else {
    a.a0_codes = w->down_codes;
    a.a0_scales = w->down_scales;
    a.b_codes = c.ws + c.L.qh;
    a.b_scales = reinterpret_cast<const float*>(c.ws + c.L.sh);
    a.K = w->f;
    a.rows_per_expert = w->d;
  }
  return a;
}

}  // namespace

int moe_ffn_prepare(const uint16_t* x_bf16, int T, int k, const moe_weights_t* w,
                    const int32_t* offsets, const int32_t* perm, void* ws, size_t ws_bytes,
                    void* stream) {
  FfnCtx c;
  int rc = ffn_check(T, k, w, ws, ws_bytes, c);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !offsets || !perm) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(x_bf16, 16)) return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if (c.gemv) {  // the token's codes (row 0 of qx) and the list of active experts
    cudaError_t e = launch_quant_rows(
        x_bf16, T, k, w->d, nullptr, 0, c.ws + c.L.qx, reinterpret_cast<float*>(c.ws + c.L.sx),
        offsets, w->E, c.nmax, reinterpret_cast<int32_t*>(c.ws + c.L.plan), nullptr, 0,
        c.di.status, static_cast<cudaStream_t>(stream), 1, t_overlap);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn prepare launch");
  }
  if (c.bg) {  // the rows in expert-sorted order and the slot plan
    cudaError_t e = launch_quant_rows(
        x_bf16, T, k, w->d, perm, T * k, c.ws + c.L.qx, reinterpret_cast<float*>(c.ws + c.L.sx),
        offsets, w->E, c.nmax, reinterpret_cast<int32_t*>(c.ws + c.L.plan), nullptr, 0,
        c.di.status, static_cast<cudaStream_t>(stream), 2, t_overlap);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn prepare launch");
  }
  cudaError_t e = launch_quant_rows(
      x_bf16, T, k, w->d, perm, T * k, c.ws + c.L.qx, reinterpret_cast<float*>(c.ws + c.L.sx),
      offsets, w->E, c.nmax, reinterpret_cast<int32_t*>(c.ws + c.L.plan),
      reinterpret_cast<int*>(c.ws + c.L.counters), c.L.n_counters, c.di.status,
      static_cast<cudaStream_t>(stream), 0, t_overlap, reinterpret_cast<int32_t*>(c.ws + c.L.ipos));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn prepare launch");
}

int moe_ffn_gate_up(int T, int k, const moe_weights_t* w, void* ws, size_t ws_bytes,
                    void* stream) {
  FfnCtx c;
  int rc = ffn_check(T, k, w, ws, ws_bytes, c);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  if (c.gemv) {
    GemvLaunch a = gemv_args(T, k, w, c);
    a.a0_codes = w->gate_codes;
    a.a0_scales = w->gate_scales;
    a.a1_codes = w->up_codes;
    a.a1_scales = w->up_scales;
    cudaError_t e = launch_gemv(1, a, static_cast<cudaStream_t>(stream), c.di.sms);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn gate/up launch");
  }
  if (c.bg) {
    BgLaunch a = bg_args(T, k, w, c);
    a.a0_codes = w->gate_codes;
    a.a0_scales = w->gate_scales;
    a.a1_codes = w->up_codes;
    a.a1_scales = w->up_scales;
    a.act = c.ws + c.L.qx;
    a.act_scales = reinterpret_cast<const float*>(c.ws + c.L.sx);
    cudaError_t e = launch_bgemv(1, a, static_cast<cudaStream_t>(stream), c.di.sms);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn gate/up launch");
  }
  cudaError_t e = launch_ffn(1, c.nmax, ffn_args(1, T, k, w, c),
                             static_cast<cudaStream_t>(stream), c.di.sms);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn gate/up launch");
}

int moe_ffn_down(int T, int k, const moe_weights_t* w, float* y_routed, float* y_shared,
                 void* ws, size_t ws_bytes, void* stream) {
  FfnCtx c;
  int rc = ffn_check(T, k, w, ws, ws_bytes, c);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  if (!y_routed || !y_shared) return fail(MOE_ERR_INVALID_ARG, "NULL output pointer");
  if (!aligned(y_routed, 16) || !aligned(y_shared, 16))
    return fail(MOE_ERR_INVALID_ARG, "outputs must be 16-byte aligned");
  if (c.gemv) {
    GemvLaunch g = gemv_args(T, k, w, c);
    g.a0_codes = w->down_codes;
    g.a0_scales = w->down_scales;
    g.y_routed = y_routed;
    g.y_shared = y_shared;
    cudaError_t e = launch_gemv(2, g, static_cast<cudaStream_t>(stream), c.di.sms);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn down launch");
  }
  if (c.bg) {  // re-quantise h, then the down GEMV
    const int R = T * k + T;
    cudaError_t e = launch_quant_h(reinterpret_cast<const float*>(c.ws + c.L.hbuf), R, w->f,
                                   c.ws + c.L.qh, reinterpret_cast<float*>(c.ws + c.L.sh),
                                   static_cast<cudaStream_t>(stream), t_overlap);
    if (e != cudaSuccess) return cuda_fail(e, "ffn h quantisation launch");
    BgLaunch b = bg_args(T, k, w, c);
    b.a0_codes = w->down_codes;
    b.a0_scales = w->down_scales;
    b.act = c.ws + c.L.qh;
    b.act_scales = reinterpret_cast<const float*>(c.ws + c.L.sh);
    b.y_routed = y_routed;
    b.y_shared = y_shared;
    b.overlap = true;  // follows the quantisation kernel of this call
    e = launch_bgemv(2, b, static_cast<cudaStream_t>(stream), c.di.sms);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn down launch");
  }
  FfnArgs a = ffn_args(2, T, k, w, c);
  a.y_routed = y_routed;
  a.y_shared = y_shared;
  cudaError_t e = launch_ffn(2, c.nmax, a, static_cast<cudaStream_t>(stream), c.di.sms);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ffn down launch");
}

namespace {

DecodeLaunch decode_args(int k, const moe_weights_t* w, const FfnCtx& c) {
  DecodeLaunch a{};
  a.gate_codes = w->gate_codes;
  a.gate_scales = w->gate_scales;
  a.up_codes = w->up_codes;
  a.up_scales = w->up_scales;
  a.down_codes = w->down_codes;
  a.down_scales = w->down_scales;
  a.qx = c.ws + c.L.qx;
  a.sx = reinterpret_cast<float*>(c.ws + c.L.sx);
  a.qh = c.ws + c.L.qh;
  a.sh = reinterpret_cast<float*>(c.ws + c.L.sh);
  a.hbuf = reinterpret_cast<float*>(c.ws + c.L.hbuf);
  a.done2 = reinterpret_cast<int*>(c.ws + c.L.done2);
  a.tc_ws = c.tc ? c.ws + c.L.dtc : nullptr;
  a.E = w->E;
  a.k = k;
  a.d = w->d;
  a.f = w->f;
  a.wait_ns = g_wait_ns.load();
  a.status = c.di.status;
  a.stall = g_stall.load();
  return a;
}

}  // namespace

int moe_ffn_path(int T, int k, const moe_weights_t* w) {
  FfnCtx c;
  const int rc = ffn_check(T, k, w, nullptr, (size_t)-1, c);  // no workspace: a query
  if (rc) return rc;
  if (T == 1 && c.fused) return MOE_PATH_SINGLE;
  if (c.bg) return MOE_PATH_BATCHED;
  return MOE_PATH_TILES;
}

int moe_forward_path(int T, int k, const moe_weights_t* w) {
  FfnCtx c;
  const int rc = ffn_check(T, k, w, nullptr, (size_t)-1, c);
  if (rc) return rc;
  if (T == 1 && c.fused && c.tc && k <= 32) return MOE_PATH_SINGLE_TC;
  return moe_ffn_path(T, k, w);
}

int moe_expert_ffn(const uint16_t* x_bf16, int T, int k, const moe_weights_t* w,
                   const int32_t* offsets, const int32_t* perm, float* y_routed, float* y_shared,
                   void* ws, size_t ws_bytes, void* stream) {
  FfnCtx c;
  int rc = ffn_check(T, k, w, ws, ws_bytes, c);
  if (rc) return rc;
  if (T > 0 && c.fused) {  // one token: the whole FFN in one kernel
    if (!x_bf16 || !offsets || !perm || !y_routed || !y_shared)
      return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(x_bf16, 16) || !aligned(y_routed, 16) || !aligned(y_shared, 16))
      return fail(MOE_ERR_INVALID_ARG, "x and the outputs must be 16-byte aligned");
    DecodeLaunch a = decode_args(k, w, c);
    a.forward = false;
    a.x = x_bf16;
    a.offsets_in = offsets;
    a.y_routed = y_routed;
    a.y_shared = y_shared;
    cudaError_t e = launch_decode(a, static_cast<cudaStream_t>(stream), c.di.sms);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "single-token ffn launch");
  }
  rc = moe_ffn_prepare(x_bf16, T, k, w, offsets, perm, ws, ws_bytes, stream);
  if (rc) return rc;
  // gate/up and down follow a kernel of this call on the stream: they may start while it
  // finishes (their prologue overlaps its tail)
  OverlapScope guard;
  rc = moe_ffn_gate_up(T, k, w, ws, ws_bytes, stream);
  if (rc) return rc;
  return moe_ffn_down(T, k, w, y_routed, y_shared, ws, ws_bytes, stream);
}

int moe_forward(const float* scores, const uint16_t* x_bf16, int T, int k,
                const moe_weights_t* w, int32_t* topk_idx, float* topk_w, int32_t* counts,
                int32_t* offsets, int32_t* perm, int32_t* pos, float* y_routed, float* y_shared,
                float* out, void* ws, size_t ws_bytes, void* stream) {
  FfnCtx c;
  int rc = ffn_check(T, k, w, ws, ws_bytes, c);
  if (rc) return rc;
  if (k > 32) return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, min(E, 32)]", k);
  if (T > 0 && c.fused) {  // one token: the whole layer in one kernel
    if (!scores || !x_bf16 || !topk_idx || !topk_w || !counts || !offsets || !perm || !pos ||
        !y_routed || !y_shared || !out)
      return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(scores, 4) || !aligned(x_bf16, 16) || !aligned(y_routed, 16) ||
        !aligned(y_shared, 16) || !aligned(out, 16) || !aligned(topk_idx, 4) ||
        !aligned(topk_w, 4) || !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(perm, 4) ||
        !aligned(pos, 4))
      return fail(MOE_ERR_INVALID_ARG, "misaligned pointer");
    DecodeLaunch a = decode_args(k, w, c);
    a.forward = true;
    a.scores = scores;
    a.x = x_bf16;
    a.idx = topk_idx;
    a.w_out = topk_w;
    a.counts = counts;
    a.offsets = offsets;
    a.perm = perm;
    a.pos = pos;
    a.y_routed = y_routed;
    a.y_shared = y_shared;
    a.out = out;
    cudaError_t e = launch_decode(a, static_cast<cudaStream_t>(stream), c.di.sms);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "single-token layer launch");
  }
  // otherwise the four calls; every kernel after the first may start under its
  // predecessor's tail
  rc = moe_route_topk(scores, T, w->E, k, topk_idx, topk_w, stream);
  if (rc) return rc;
  OverlapScope guard;
  rc = moe_dispatch(topk_idx, T, k, w->E, counts, offsets, perm, pos, c.ws + c.L.dispatch,
                    dispatch_ws_bytes(T, k, w->E), stream);
  if (rc) return rc;
  rc = moe_expert_ffn(x_bf16, T, k, w, offsets, perm, y_routed, y_shared, ws, ws_bytes, stream);
  if (rc) return rc;
  return moe_combine(y_routed, y_shared, topk_w, pos, T, k, w->d, out, stream);
}

int moe_forward_q2(const float* scores, const uint16_t* x_bf16, int k, const moe_weights_t* w,
                   const moe_q2_experts_t* q2, int32_t* topk_idx, float* topk_w,
                   int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                   float* y_routed, float* y_shared, float* out, void* ws, size_t ws_bytes,
                   void* stream) {
  if (!q2) return fail(MOE_ERR_INVALID_ARG, "NULL 2-bit expert descriptor");
  FfnCtx c;
  int rc = ffn_check(1, k, w, ws, ws_bytes, c);
  if (rc) return rc;
  if (k > 32) return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, min(E, 32)]", k);
  if (w->d % 2048 || w->f % 2048)
    return fail(MOE_ERR_INVALID_ARG, "d=%d, f=%d must be multiples of 2048", w->d, w->f);
  if (!q2->gate_codes || !q2->gate_scales || !q2->up_codes || !q2->up_scales ||
      !q2->down_codes || !q2->down_scales)
    return fail(MOE_ERR_INVALID_ARG, "NULL 2-bit weight pointer");
  if (!aligned(q2->gate_codes, 16) || !aligned(q2->up_codes, 16) || !aligned(q2->down_codes, 16) ||
      !aligned(q2->gate_scales, 16) || !aligned(q2->up_scales, 16) || !aligned(q2->down_scales, 16) ||
      !aligned(w->gate_scales, 16) || !aligned(w->up_scales, 16) || !aligned(w->down_scales, 16))
    return fail(MOE_ERR_INVALID_ARG, "weight arrays must be 16-byte aligned");
  if (!scores || !x_bf16 || !topk_idx || !topk_w || !counts || !offsets || !perm || !pos ||
      !y_routed || !y_shared || !out)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(scores, 4) || !aligned(x_bf16, 16) || !aligned(y_routed, 16) ||
      !aligned(y_shared, 16) || !aligned(out, 16) || !aligned(topk_idx, 4) ||
      !aligned(topk_w, 4) || !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(perm, 4) ||
      !aligned(pos, 4))
    return fail(MOE_ERR_INVALID_ARG, "misaligned pointer");
  int max_smem = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int ctas = c.di.sms < kMaxCtas ? c.di.sms : kMaxCtas;
  if (!decode_fits(k, w->d, w->f, ctas, true) ||
      decode_smem_bytes(w->d, w->f, true) > (size_t)max_smem)
    return fail(MOE_ERR_INVALID_ARG, "shape (k=%d, d=%d, f=%d) does not fit the single-token kernel",
                k, w->d, w->f);
  DecodeLaunch a = decode_args(k, w, c);
  a.forward = true;
  a.scores = scores;
  a.x = x_bf16;
  a.idx = topk_idx;
  a.w_out = topk_w;
  a.counts = counts;
  a.offsets = offsets;
  a.perm = perm;
  a.pos = pos;
  a.y_routed = y_routed;
  a.y_shared = y_shared;
  a.out = out;
  a.q2_gate_codes = q2->gate_codes;
  a.q2_gate_scales = q2->gate_scales;
  a.q2_up_codes = q2->up_codes;
  a.q2_up_scales = q2->up_scales;
  a.q2_down_codes = q2->down_codes;
  a.q2_down_scales = q2->down_scales;
  cudaError_t e = launch_decode(a, static_cast<cudaStream_t>(stream), c.di.sms);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "single-token 2-bit layer launch");
}

size_t moe_fp8_gemm_workspace_size(int M, int N, int K) {
  if (M < 1 || M > 64 || N < 128 || N % 128 || K < 512 || K % 512) return 0;
  return fp8_gemm_ws_bytes(M, N, K, false);
}

int moe_fp8_gemm(const uint8_t* A, const float* sa, int M, int K, const uint8_t* B,
                 const float* sb, int N, float* C, void* ws, size_t ws_bytes, void* stream) {
  if (M < 0 || M > 64) return fail(MOE_ERR_INVALID_ARG, "M=%d outside [0, 64]", M);
  if (N < 128 || N % 128 || K < 512 || K % 512)
    return fail(MOE_ERR_INVALID_ARG, "N=%d must be a multiple of 128, K=%d of 512", N, K);
  if (M == 0) return MOE_OK;
  if (!A || !sa || !B || !sb || !C || !ws) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 8) || !aligned(sa, 4) ||
      !aligned(sb, 4) || !aligned(ws, 256))
    return fail(MOE_ERR_INVALID_ARG, "A, B 16-byte, C 8-byte, ws 256-byte aligned");
  const size_t need = fp8_gemm_ws_bytes(M, N, K, false);
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  DeviceInfo di;
  int rc = device_info(di);
  if (rc) return rc;
  Fp8Launch a{};
  a.A = A;
  a.sa = sa;
  a.B0 = B;
  a.sb0 = sb;
  a.M = M;
  a.N = N;
  a.K = K;
  a.C = C;
  a.ws = static_cast<uint8_t*>(ws);
  a.zero_counters = true;
  cudaError_t e = launch_fp8_gemm(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "fp8_gemm launch");
}

namespace {
// workspace of moe_shared_expert_fp8: qx, sx, h, qh, sh, then each GEMM's partials and
// counters (separate regions: a counter must not sit in the other GEMM's partials)
struct SharedFp8Layout {
  size_t qx, sx, h, qh, sh, g1, g2, cnt, total;
};
SharedFp8Layout shared_fp8_layout(int T, int d, int f) {
  SharedFp8Layout L{};
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t o = 0;
  L.qx = o; o = up(o + (size_t)T * d);
  L.sx = o; o = up(o + (size_t)T * (d / 128) * 4);
  L.h = o;  o = up(o + (size_t)T * f * 4);
  L.qh = o; o = up(o + (size_t)T * f);
  L.sh = o; o = up(o + (size_t)T * (f / 128) * 4);
  L.g1 = o; o = up(o + fp8_gemm_ws_bytes(T, f, d, true));
  L.g2 = o; o = up(o + fp8_gemm_ws_bytes(T, d, f, false));
  L.cnt = o; o = up(o + (fp8_gemm_counters(f, true) + fp8_gemm_counters(d, false)) * sizeof(int));
  L.total = o;
  return L;
}
}  // namespace

int moe_shared_expert_fp8_offsets(int T, int d, int f, size_t off[5]) {
  if (!off) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (T < 1 || T > 64 || d < 512 || d % 512 || f < 512 || f % 512)
    return fail(MOE_ERR_INVALID_ARG, "T=%d, d=%d, f=%d outside the accepted shapes", T, d, f);
  const SharedFp8Layout L = shared_fp8_layout(T, d, f);
  off[0] = L.qx;
  off[1] = L.sx;
  off[2] = L.h;
  off[3] = L.qh;
  off[4] = L.sh;
  return MOE_OK;
}

size_t moe_shared_expert_fp8_workspace_size(int T, int d, int f) {
  if (T < 1 || T > 64 || d < 512 || d % 512 || f < 512 || f % 512) return 0;
  return shared_fp8_layout(T, d, f).total;
}

int moe_shared_expert_fp8(const uint16_t* x_bf16, int T, const moe_fp8_expert_t* w,
                          float* y_shared, void* ws, size_t ws_bytes, void* stream) {
  if (!w) return fail(MOE_ERR_INVALID_ARG, "NULL weights");
  const int d = w->d, f = w->f;
  if (T < 0 || T > 64) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [0, 64]", T);
  if (d < 512 || d % 512 || f < 512 || f % 512)
    return fail(MOE_ERR_INVALID_ARG, "d=%d, f=%d must be multiples of 512", d, f);
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !y_shared || !ws || !w->gate || !w->up || !w->down || !w->gate_scales ||
      !w->up_scales || !w->down_scales)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(x_bf16, 16) || !aligned(y_shared, 8) || !aligned(ws, 256) ||
      !aligned(w->gate, 16) || !aligned(w->up, 16) || !aligned(w->down, 16))
    return fail(MOE_ERR_INVALID_ARG, "misaligned pointer");
  const SharedFp8Layout L = shared_fp8_layout(T, d, f);
  if (ws_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  DeviceInfo di;
  int rc = device_info(di);
  if (rc) return rc;
  uint8_t* base = static_cast<uint8_t*>(ws);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* qx = base + L.qx;
  float* sx = reinterpret_cast<float*>(base + L.sx);
  float* h = reinterpret_cast<float*>(base + L.h);
  uint8_t* qh = base + L.qh;
  float* sh = reinterpret_cast<float*>(base + L.sh);
  // both GEMMs' counters in one clear; every launch leaves its counters zero again
  int* cnt = reinterpret_cast<int*>(base + L.cnt);
  const size_t n1 = fp8_gemm_counters(f, true), n2 = fp8_gemm_counters(d, false);
  cudaError_t e = cudaMemsetAsync(cnt, 0, (n1 + n2) * sizeof(int), s);
  if (e == cudaSuccess)
    e = launch_quant_rows(x_bf16, T, 1, d, nullptr, 0, qx, sx, nullptr, 0, 0, nullptr, nullptr, 0,
                          di.status, s);
  Fp8Launch a{};
  a.A = qx;
  a.sa = sx;
  a.B0 = w->gate;
  a.sb0 = w->gate_scales;
  a.B1 = w->up;
  a.sb1 = w->up_scales;
  a.M = T;
  a.N = f;
  a.K = d;
  a.C = h;
  a.ws = base + L.g1;
  a.cnt = cnt;
  a.overlap = true;
  if (e == cudaSuccess) e = launch_fp8_gemm(a, s);
  if (e == cudaSuccess) e = launch_quant_h(h, T, f, qh, sh, s, true);
  Fp8Launch b{};
  b.A = qh;
  b.sa = sh;
  b.B0 = w->down;
  b.sb0 = w->down_scales;
  b.M = T;
  b.N = d;
  b.K = f;
  b.C = y_shared;
  b.ws = base + L.g2;
  b.cnt = cnt + n1;
  b.overlap = true;
  if (e == cudaSuccess) e = launch_fp8_gemm(b, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "shared expert fp8 launch");
}

int moe_expert_cache_reset(const moe_expert_cache_t* c, void* stream) {
  if (!c || !c->slot_of || !c->expert_of || !c->last_use || !c->clock || !c->stats || !c->fetch)
    return fail(MOE_ERR_INVALID_ARG, "NULL cache pointer");
  if (c->E < 1 || c->slots.E < 1) return fail(MOE_ERR_INVALID_ARG, "E=%d, S=%d", c->E, c->slots.E);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(c->slot_of, 0xFF, (size_t)c->E * sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->expert_of, 0xFF, (size_t)c->slots.E * sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->last_use, 0, (size_t)c->slots.E * sizeof(int64_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->clock, 0, sizeof(int64_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->stats, 0, 2 * sizeof(int64_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->fetch, 0, sizeof(int32_t), s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "cache reset");
}

int moe_forward_streamed(const float* scores, const uint16_t* x_bf16, int k,
                         const moe_host_experts_t* host, const moe_expert_cache_t* cache,
                         int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                         int32_t* perm, int32_t* pos, float* y_routed, float* y_shared,
                         float* out, void* ws, size_t ws_bytes, void* stream) {
  if (!host || !cache) return fail(MOE_ERR_INVALID_ARG, "NULL descriptor");
  const moe_weights_t& sl = cache->slots;
  const int E = cache->E, S = sl.E;
  if (k < 1 || k > 32 || k > S || k > E)
    return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, min(32, S=%d, E=%d)]", k, S, E);
  // the routed view: E experts scored and routed, workspace laid out for them
  moe_weights_t wr = sl;
  wr.E = E;
  FfnCtx c;
  int rc = ffn_check(1, k, &wr, ws, ws_bytes, c);
  if (rc) return rc;
  if (!c.fused)
    return fail(MOE_ERR_INVALID_ARG, "shape (k=%d, d=%d, f=%d) does not fit the single-token kernel",
                k, sl.d, sl.f);
  if (!host->gate_codes || !host->gate_scales || !host->up_codes || !host->up_scales ||
      !host->down_codes || !host->down_scales || !cache->slot_of || !cache->expert_of ||
      !cache->last_use || !cache->clock || !cache->fetch || !cache->stats)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  const uint8_t* src[6] = {host->gate_codes, host->gate_scales, host->up_codes, host->up_scales,
                           host->down_codes, host->down_scales};
  uint8_t* dst[6] = {const_cast<uint8_t*>(sl.gate_codes), const_cast<uint8_t*>(sl.gate_scales),
                     const_cast<uint8_t*>(sl.up_codes), const_cast<uint8_t*>(sl.up_scales),
                     const_cast<uint8_t*>(sl.down_codes), const_cast<uint8_t*>(sl.down_scales)};
  const long long d = sl.d, f = sl.f;
  const long long bytes[6] = {f * d / 2, f * d / 32, f * d / 2, f * d / 32, d * f / 2, d * f / 32};
  for (int a = 0; a < 6; ++a) {
    if (!aligned(src[a], 16) || !aligned(dst[a], 16))
      return fail(MOE_ERR_INVALID_ARG, "expert arrays must be 16-byte aligned");
    // the copy kernel reads the host arrays directly: they must be pinned host memory that
    // the device addresses at the same pointer (unified addressing), not pageable memory
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, src[a]) != cudaSuccess || at.type != cudaMemoryTypeHost ||
        at.devicePointer != src[a]) {
      cudaGetLastError();
      return fail(MOE_ERR_INVALID_ARG, "host expert array %d is not pinned, device-mapped memory", a);
    }
  }
  if (!x_bf16 || !counts || !offsets || !perm || !pos || !y_routed || !y_shared || !out)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(x_bf16, 16) || !aligned(y_routed, 16) || !aligned(y_shared, 16) || !aligned(out, 16))
    return fail(MOE_ERR_INVALID_ARG, "misaligned pointer");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = moe_route_topk(scores, 1, E, k, topk_idx, topk_w, stream);
  if (rc) return rc;
  cudaError_t e = launch_cache(topk_idx, k, S, cache->slot_of, cache->expert_of,
                               reinterpret_cast<long long*>(cache->last_use),
                               reinterpret_cast<long long*>(cache->clock), cache->fetch,
                               reinterpret_cast<long long*>(cache->stats), c.di.status, s);
  if (e == cudaSuccess) e = launch_fetch(src, dst, bytes, cache->fetch, c.di.sms, s);
  if (e != cudaSuccess) return cuda_fail(e, "expert cache launch");
  DecodeLaunch a = decode_args(k, &wr, c);
  a.forward = true;
  a.scores = scores;
  a.x = x_bf16;
  a.idx = topk_idx;
  a.w_out = topk_w;
  a.counts = counts;
  a.offsets = offsets;
  a.perm = perm;
  a.pos = pos;
  a.y_routed = y_routed;
  a.y_shared = y_shared;
  a.out = out;
  a.slot_of = cache->slot_of;
  a.maps_E = S;
  e = launch_decode(a, s, c.di.sms);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "single-token streamed layer launch");
}

int moe_combine(const float* y_routed, const float* y_shared, const float* topk_w,
                const int32_t* pos, int T, int k, int d, float* out, void* stream) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d < 0", T);
  if (k < 1 || k > 32) return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, 32]", k);
  if (d < 4 || d % 4) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 4", d);
  if (T == 0) return MOE_OK;
  if (!y_routed || !y_shared || !topk_w || !pos || !out)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(y_routed, 16) || !aligned(y_shared, 16) || !aligned(out, 16))
    return fail(MOE_ERR_INVALID_ARG, "y_routed, y_shared and out must be 16-byte aligned");
  DeviceInfo di;
  int rc = device_info(di);
  if (rc) return rc;
  cudaError_t e = launch_combine(y_routed, y_shared, topk_w, pos, T, k, d, out, di.status,
                                 static_cast<cudaStream_t>(stream), t_overlap);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "combine launch");
}

}  // extern "C"
