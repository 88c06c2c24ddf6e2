// Internal declarations shared by the bitmoe CUDA sources (not part of the C ABI).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace bitmoe {

// Division by a divisor fixed for a launch, as a multiply-high, an add and a shift (the
// round-up method of Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1,
// n / d = (umulhi(n, m) + n) >> s for 1 <= d < 2^31 and 0 <= n < 2^31 (the sum stays
// below 2^32).  The kernels' per-stage work splits divide by runtime sizes; an integer
// division there costs tens of instructions on every warp's path.
struct FastDiv {
  uint32_t d, m, s;
  __host__ __device__ constexpr explicit FastDiv(uint32_t d_ = 1) : d(d_ < 1 ? 1 : d_), m(0), s(0) {
    while ((1ull << s) < d) ++s;
    m = (uint32_t)(((1ull << 32) * ((1ull << s) - d)) / d + 1);
  }
  __host__ __device__ __forceinline__ int div(int n) const {
#ifdef __CUDA_ARCH__
    const uint32_t hi = __umulhi((uint32_t)n, m);
#else
    const uint32_t hi = (uint32_t)(((uint64_t)(uint32_t)n * m) >> 32);
#endif
    return (int)((hi + (uint32_t)n) >> s);
  }
};

// Device-side status word (one per device): bit 0 = a bounded wait expired,
// bit 1 = an expert id outside [0, E) reached the dispatch kernel (or a plan entry was
// out of range).
constexpr int kStatusTimeout = 1;
constexpr int kStatusBadIndex = 2;

// Token tiles of the expert FFN: every expert's rows (routed pairs in expert-sorted
// order, then the T shared-expert rows) are cut into tiles of at most kNmax rows.
// Up to T = 64 most experts get a few tokens, and tiles of 32 tokens x 256 weight rows
// stream twice the weight bytes per pipeline stage of 112 x 128 tiles (measured at T = 64
// with Zipf(1.0) routing: 544 vs 840 us per layer).
constexpr int kNmaxLarge = 112;  // T > 64
constexpr int kNmaxSmall = 32;   // T <= 64
constexpr int kSmallTileMaxT = 64;
inline int nmax_for(int T) { return T <= kSmallTileMaxT ? kNmaxSmall : kNmaxLarge; }
// Widest token tile a launch can see (a tile never holds more rows than T).
inline int ncap_for(int T) { return T < nmax_for(T) ? T : nmax_for(T); }

// The FFN kernels run at most this many CTAs (one per SM); the stream-K partial slots of
// the workspace are sized for it.
constexpr int kMaxCtas = 148;

// Plan layout (int32 words in the workspace):
//   [0, E+2)              ttbase: first token tile of expert e (e = 0..E), ttbase[E+1] = total
//   [E+2, E+2 + 2*ntmax)  tiles: (row0, n) per token tile
inline size_t plan_ntmax(int R, int E) { return (size_t)R / 16 + (size_t)E + 2; }

// Single-token batches (T = 1) run the expert FFN as FP4 GEMV kernels (decode.cu, gemv.cu)
// when the shapes allow it; batches up to kBgMaxT run the batched FP4 GEMV (bgemv.cu);
// larger ones use the tcgen05 tile kernels (ffn.cu).
constexpr int kGemvMaxT = 1;
constexpr int kBgMaxT = 64;
constexpr int kBgSlotTokens = 8;  // tokens per slot of the batched GEMV (the MMA's N)

struct WorkspaceLayout {
  size_t plan, qx, sx, qh, sh, counters, partials, hbuf, done2, dtc, dispatch, ipos, total;
  size_t n_counters;
};
WorkspaceLayout workspace_layout(int T, int k, int E, int d, int f);

// Host launchers (each returns a cudaError_t of the launch)
cudaError_t launch_route_topk(const float* scores, int T, int E, int k, int32_t* idx, float* w,
                              cudaStream_t s, bool overlap = false);
// scores [T][E] fp32 = x [T][d] bf16 . W_router [E][d] bf16 (router.cu)
cudaError_t launch_router(const uint16_t* x, const uint16_t* w, int T, int d, int E, float* scores,
                          cudaStream_t s, bool overlap = false);
cudaError_t launch_dispatch(const int32_t* idx, int T, int k, int E, int32_t* counts,
                            int32_t* offsets, int32_t* perm, int32_t* pos, int* status,
                            cudaStream_t s, bool overlap = false);
// Multi-CTA dispatch for large batches (T*k >= kDispatchMultiMin pairs): its workspace
// holds one count per (segment of pairs, expert); 0 below the threshold.
constexpr long long kDispatchMultiMin = 8192;
size_t dispatch_ws_bytes(int T, int k, int E);
cudaError_t launch_dispatch_multi(const int32_t* idx, int T, int k, int E, int32_t* counts,
                                  int32_t* offsets, int32_t* perm, int32_t* pos, int32_t* cnt,
                                  int* status, cudaStream_t s, bool overlap);
// rows r < P = T*k take token perm[r]/k, rows P <= r < P+T take token r-P; perm may be
// NULL with P = 0 for a plain quantisation of T rows.  If plan != NULL, one extra block
// writes the token-tile plan (plan_mode 0), the single-token path's list of active
// experts (plan_mode 1) or the batched path's slot plan (plan_mode 2).  With perm and
// ipos (T*k ints of scratch), from kQuantTokensMinPairs pairs, each token is quantised
// once and its codes written to all its rows: a launch that inverts perm into ipos, then
// one block per token (4096 tokens, top-6: 30 us against 85 us for one block per row; at
// 64 tokens the second launch costs more than it saves).
constexpr int kQuantTokensMinPairs = 2048;
cudaError_t launch_quant_rows(const uint16_t* x, int T, int k, int d, const int32_t* perm,
                              int nrows_routed, uint8_t* q, float* s, const int32_t* offsets,
                              int E, int nmax, int32_t* plan, int* counters, size_t n_counters,
                              int* status, cudaStream_t st, int plan_mode = 0,
                              bool overlap = false, int32_t* ipos = nullptr);
// h [R][f] fp32 -> e4m3 codes [R][f] and scales [R][f/128] (batched GEMV path)
cudaError_t launch_quant_h(const float* h, int R, int f, uint8_t* q, float* s, cudaStream_t st,
                           bool overlap);
cudaError_t launch_combine(const float* y, const float* ysh, const float* w, const int32_t* pos,
                           int T, int k, int d, float* out, int* status, cudaStream_t s,
                           bool overlap = false);

struct FfnArgs {
  const uint8_t* a0_codes;   // gate (phase 1) or down (phase 2) codes, all experts
  const uint8_t* a0_scales;
  const uint8_t* a1_codes;   // up (phase 1 only)
  const uint8_t* a1_scales;
  const uint8_t* b_codes;    // qx (phase 1) or qh (phase 2) rows [R][K]
  const float* b_scales;     // sx or sh [R][K/128]
  const int32_t* plan;
  int E, K, rows_per_expert, R, P;
  uint8_t* qh;               // phase 1 outputs
  float* sh;
  int f;
  float* y_routed;           // phase 2 outputs
  float* y_shared;
  int d;
  long long wait_ns;
  int* status;
  int* counters;             // stream-K fix-up counters (zeroed by the prepare kernel)
  float* partials;           // stream-K partial slots
  int ncap;                  // widest token tile
  int l2_hints;              // bit 0: weight boxes evict-first; bit 1: activation boxes evict-last
  bool overlap;              // launch as a dependent of the previous kernel (see launch_pdl)
};
cudaError_t launch_ffn(int phase, int nmax, const FfnArgs& a, cudaStream_t s, int num_sms);
// dynamic shared memory of a launch
size_t ffn_smem_bytes(int phase, int nmax, int E, int rows_per_expert);

// Single-token FP4 GEMV path (gemv.cu).  The plan holds the active experts (routed
// ones with a token, in ascending id, then the shared expert E) as (expert, output row)
// pairs after their count; the output row is the routed row in expert-sorted order, or
// -1 for the shared expert.
struct GemvLaunch {
  const uint8_t* a0_codes;   // gate (phase 1) or down (phase 2)
  const uint8_t* a0_scales;
  const uint8_t* a1_codes;   // up (phase 1)
  const uint8_t* a1_scales;
  const int32_t* plan;
  const uint8_t* qx;         // phase 1: the token's e4m3 codes [d] and block scales
  const float* sx;
  float* hbuf;               // h [active experts][f] fp32
  float* y_routed;
  float* y_shared;
  uint8_t* qh;               // re-quantised h [row][f] and scales [row][f/128]
  float* sh;
  int E, d, f, P;
  long long wait_ns;
  int* status;
  int stall;                 // test knob (moe_set_test_stall)
  bool overlap;
};
cudaError_t launch_gemv(int phase, const GemvLaunch& a, cudaStream_t s, int num_sms);
size_t gemv_smem_bytes(int phase, int K);
// a launch's units (8 h-rows in phase 1, 16 down rows in phase 2, of every active
// expert) are cut into one range per CTA of at most this many units
int gemv_max_units_per_cta();

// Batched FP4 GEMV path (bgemv.cu), 2 <= T <= kBgMaxT: phase 1 reads the activation rows
// qx/sx and writes h [R][f] fp32; phase 2 reads qh/sh and writes y.  The plan holds the
// slots (expert, first row, rows <= kBgSlotTokens) after their count.
struct BgLaunch {
  const uint8_t* a0_codes;   // gate (phase 1) or down (phase 2)
  const uint8_t* a0_scales;
  const uint8_t* a1_codes;   // up (phase 1)
  const uint8_t* a1_scales;
  const int32_t* plan;
  const uint8_t* act;        // [R][K] e4m3 rows (qx or qh)
  const float* act_scales;   // [R][K/128]
  float* hbuf;
  float* y_routed;
  float* y_shared;
  int E, d, f, P, R;
  long long wait_ns;
  int* status;
  bool overlap;
};
cudaError_t launch_bgemv(int phase, const BgLaunch& a, cudaStream_t s, int num_sms);
size_t bgemv_smem_bytes(int K);

// Single-token layer in one cooperative kernel (decode.cu): forward = routing from the
// scores, dispatch and combine included; otherwise the expert FFN from dispatch offsets.
struct DecodeLaunch {
  bool forward;
  const uint8_t* gate_codes;
  const uint8_t* gate_scales;
  const uint8_t* up_codes;
  const uint8_t* up_scales;
  const uint8_t* down_codes;
  const uint8_t* down_scales;
  const float* scores;
  const uint16_t* x;
  const int32_t* offsets_in;
  int32_t *idx, *counts, *offsets, *perm, *pos;
  float* w_out;
  float *y_routed, *y_shared, *out;
  uint8_t* qx;
  float* sx;
  uint8_t* qh;
  float* sh;
  float* hbuf;
  int* done2;
  int E, k, d, f;
  long long wait_ns;
  int* status;
  int stall;
  // Q2 form (forward only): the E routed experts in the 2-bit codec; NULL otherwise, and
  // then the FP4 arrays hold all E + 1 experts (in the Q2 form only the shared one, E)
  const uint8_t* q2_gate_codes = nullptr;
  const uint8_t* q2_gate_scales = nullptr;
  const uint8_t* q2_up_codes = nullptr;
  const uint8_t* q2_up_scales = nullptr;
  const uint8_t* q2_down_codes = nullptr;
  const uint8_t* q2_down_scales = nullptr;
  // expert cache: the FP4 arrays hold maps_E + 1 slots (the shared expert in the last);
  // routed expert e's weights are in slot slot_of[e].  maps_E < 0: the plain layout.
  const int32_t* slot_of = nullptr;
  int maps_E = -1;
  // forward, FP4: the tensor-core form of the kernel (decode_tc.cu) runs with this
  // workspace region (decode_tc_ws_bytes); NULL: the CUDA-core form (decode.cu)
  uint8_t* tc_ws = nullptr;
};
cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t s, int num_sms);
cudaError_t launch_decode_tc(const DecodeLaunch& a, cudaStream_t s, int num_sms);
// whether the tensor-core single-token kernel takes (k, d, f) on `ctas` CTAs, its shared
// memory and its workspace region
bool decode_tc_fits(int k, int d, int f, int ctas);
size_t decode_tc_smem_bytes(int d, int f);
size_t decode_tc_ws_bytes(int k, int d, int f);
cudaError_t reset_tc_barrier(int ctas);
size_t decode_smem_bytes(int d, int f, bool q2 = false);
// whether the single-token kernel's per-CTA limits hold for (k, d, f) on `ctas` CTAs
// (q2: with 2-bit routed experts)
bool decode_fits(int k, int d, int f, int ctas, bool q2 = false);
// FP8 x FP8 GEMM for M <= 64 rows of A (fp8.cu): C[m][n] = sum_kb sa[m][kb] sb[n/128][kb]
// sum_k A[m][k] B[n][k], A [M][K] and B [N][K] e4m3, sa [M][K/128], sb [N/128][K/128] fp32.
// With B1 (the up projection beside B0 = gate) C = silu(A B0^T) * (A B1^T).  K % 512 == 0,
// N % 128 == 0; the workspace holds the partial sums and the row blocks' counters, which
// must be zero on entry (zero_counters: the launch clears them first; every launch leaves
// them zero).
struct Fp8Launch {
  const uint8_t* A;
  const float* sa;
  const uint8_t* B0;
  const float* sb0;
  const uint8_t* B1;
  const float* sb1;
  int M, N, K;
  float* C;
  uint8_t* ws;
  int* cnt;            // the row blocks' counters (NULL: at the end of ws)
  bool zero_counters;
  bool overlap;
};
size_t fp8_gemm_ws_bytes(int M, int N, int K, bool fused);
size_t fp8_gemm_counters(int N, bool fused);  // counters (ints) a launch uses
cudaError_t launch_fp8_gemm(const Fp8Launch& a, cudaStream_t s);
// Expert cache (stream.cu): the LRU decisions of one token's step (one thread) and the
// copy of the listed experts from host memory into their slots.  fetch = [count, then
// (expert, slot) pairs]; stats = [hits, misses] accumulated.
cudaError_t launch_cache(const int32_t* idx, int k, int S, int32_t* slot_of, int32_t* expert_of,
                         long long* last_use, long long* clock, int32_t* fetch, long long* stats,
                         int* status, cudaStream_t s);
cudaError_t launch_fetch(const uint8_t* const src[6], uint8_t* const dst[6],
                         const long long bytes[6], const int32_t* fetch, int num_sms,
                         cudaStream_t s);
// clears the single-token kernel's grid barrier (after a reported timeout)
cudaError_t reset_grid_barrier();

// Launch, with `overlap`, as a programmatic dependent launch: the kernel may start while
// the previous kernel on the stream finishes (every kernel of this library calls
// griddep_wait() before it touches global memory, and griddep_launch_dependents() early).
// Only valid when the previous operation on the stream is one of this library's kernels:
// the wait covers prerequisite kernels, not copies or host work queued before them.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, bool overlap, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// The driver's cuTensorMapEncodeTiled (looked up once; NULL if the driver lacks it).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encode_fn();
// Tensor maps the GEMV kernels use (defined in abi.cu; false if encoding fails).
bool make_byte_map(CUtensorMap* m, const void* base, long long cols, long long rows, int box_cols,
                   int box_rows);
bool make_code_map(CUtensorMap* m, const void* base, long long cols, long long rows, int box_rows,
                   int pieces = 2);
bool make_f32_map(CUtensorMap* m, const void* base, long long cols, long long rows, int box_rows);

// Defined in abi.cu: sets the thread-local message that moe_last_error returns.
int record_error(int code, const char* msg);


}  // namespace bitmoe
