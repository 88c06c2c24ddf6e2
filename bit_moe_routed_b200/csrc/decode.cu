// Single-token decode of the whole MoE layer in one kernel: routing, dispatch, activation
// quantisation, gate/up FP4 GEMV, SwiGLU, re-quantisation, down FP4 GEMV and the
// routing-weighted combine.
//
// At T = 1 the layer is bound by reading the k + 1 selected experts' FP4 codes and block
// scales once (dpshk.com article, "核心实现三": an expert is read once for all its tokens;
// "核心实现四": FP4 decoded inside the GEMV, gate and up on one quantised input).  As
// separate kernels, the routing, dispatch, quantisation and combine steps and the
// launch gaps between them cost as much as a third of the layer (ai-muninn.com post,
// "一張 22G 老卡跑 284B": the fixed per-token cost of launches and round trips).  Here
// they run inside one cooperative launch, and every SM starts streaming weights at once:
//
//   prologue  every CTA issues the copies of its share of the shared expert (always
//             active, known before routing), then computes the top-k of the token's
//             scores (warp 0) and quantises the token (warps 1-8) redundantly, so no
//             grid-wide step precedes the weight stream; CTA 0 stores the routing,
//             dispatch and quantisation outputs;
//   phase 1   gate/up: units of 8 h-rows (8 gate + the same 8 up weight rows) x 512-wide
//             K stages, as in the two-kernel GEMV path; h = silu(g) * u to the workspace;
//   barrier   one bounded grid barrier (all h written); the down weights of each warp's
//             first phase-2 stages stream into its ring during the phase-1 tail and the
//             barrier;
//   phase 2   each CTA quantises the h of its experts (amax / 448, IEEE divide, e4m3
//             round to nearest even) and runs the down GEMV (units of 16 down rows);
//   combine   per block of 16 output rows, the last of the k + 1 experts to write it
//             sums out = y_shared + sum_j w_j y_j in fixed j order.
//
// Work split: the shared expert's units and the routed experts' units are each cut into
// one contiguous range per CTA (so every CTA holds 1-2 shared units to stream before
// routing is known), and a CTA's stages go round-robin to its 16 warps, each with a
// private ring of 3 stages filled by TMA (3-D code boxes with the 128-byte swizzle, 2-D
// scale boxes).  Per 32-element block the warp decodes e2m1 pairs to f16 in registers
// and runs two mma.sync m16n8k16 (fp32 accumulate); block partials are scaled by the
// row's ue8m0 scale (exact) and the activation's fp32 block scale, and each row's stage
// partials are summed in K order after a CTA barrier: results do not depend on timing and
// equal those of the two-kernel path bit for bit.
//
// 2-bit routed experts (the Q2 form, moe_forward_q2): the deployed model of the
// ai-muninn.com post ("一張 22G 老卡跑 284B") keeps its routed experts at 2 bits per weight
// (IQ2_XXS, 2.0625 bpw) and the shared expert at higher precision.  In this form the
// routed experts' units stream a 2-bit codec (four codes per byte, value code - 1.5, one
// ue8m0 scale per 128 elements) while the shared expert stays FP4.  A 2-bit stage holds
// the same 4 KB of codes per 16 rows as an FP4 stage but 1024 elements per row; per
// 128-element chunk a lane turns its 2 x 16 codes of rows g and g + 8 into e4m3 bytes with
// byte permutes (a 4-entry table indexed by the codes) and runs four mma.sync m16n8k32
// e4m3 against the token's e4m3 codes, accumulating the chunk's 128 products in the
// tensor core, then applies the chunk's ue8m0 weight scale (exact) and the token's fp32
// block scale.  A shared unit counts twice in the work split (twice the stages).
//
// Every wait is bounded (%globaltimer): an expired wait records MOE_ERR_TIMEOUT in the
// status word, the CTA skips its remaining work, lets its issued copies land, still
// takes part in the grid barrier and returns.
#include "internal.cuh"
#include "ptx.cuh"
#include "single_token.cuh"
#include "waits.cuh"

#include <cstring>
#include <type_traits>

namespace bitmoe {

// Grid barrier of the single-token kernel, one per device (zero when the module loads):
// the count of CTA arrivals, a multiple of G between barriers.  A CTA that adds 1 to n
// waits until the count reaches the next multiple of G above n, so the last arrival's own
// add opens the barrier (one atomic round trip).  It serves one launch at a time: a launch
// holds every SM (one CTA per SM, by its shared memory) until all its CTAs have passed the
// barrier, so a later launch's CTAs cannot arrive before the barrier has opened.
__device__ unsigned long long g_grid_bar;

namespace {

// 16 warps x 3 ring stages: the same 204 KB in flight per SM as 24 x 2, and room for 128
// registers per thread, so the inner loop does not spill (measured: 34.9 vs 37.0 us per
// decode layer at d = 4096, f = 2048, k = 6)
constexpr int kDcWarps = 16;
constexpr int kDcThreads = kDcWarps * 32;
constexpr int kDcStages = 3;                       // ring depth per warp
constexpr int kDcRows = 16;                        // weight rows per stage
constexpr int kDcCodeBytes = kDcRows * 256;        // 512 FP4 elements per row
constexpr int kDcScaleBytes = kDcRows * 16;        // 16 ue8m0 bytes per row
constexpr int kDcStageBytes = kDcCodeBytes + kDcScaleBytes;
constexpr int kDcMaxUnits = 16;                    // units per CTA and phase
constexpr int kDcMaxSlots = 33;                    // active experts (k <= 32) + shared
constexpr int kDcP2Slots = 3;                      // experts whose h a CTA holds in phase 2

enum { kModeForward = 0, kModeFfn = 1 };

struct DecodeParams {
  CUtensorMap tm_gc, tm_gs, tm_uc, tm_us, tm_dc, tm_ds;  // codes (3-D) and scales (2-D)
  CUtensorMap tm_gq, tm_gqs, tm_uq, tm_uqs, tm_dq, tm_dqs;  // 2-bit routed experts (Q2 form)
  const float* scores;        // forward: [E] router scores
  const uint16_t* x;          // [d] bf16 token
  const int32_t* offsets_in;  // ffn: [E+1] from moe_dispatch
  int32_t* idx;               // forward outputs: [k], [k], [E], [E+1], [k], [k]
  float* w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* pos;
  float* y_routed;            // [k][d], row = pair's sorted position
  float* y_shared;            // [d]
  float* out;                 // forward: [d]
  uint8_t* qx;                // workspace: the token's codes [d] and scales [d/128]
  float* sx;
  uint8_t* qh;                // workspace: re-quantised h [k+1][f], scales [k+1][f/128]
  float* sh;
  float* hbuf;                // workspace: h [active experts][f] fp32 (shared last)
  int* done2;                 // workspace: [d/16] combine counters (forward)
  int E, k, d, f;
  long long wait_ns;
  int* status;
  int stall;
  // weight rows: expert e's are at slot_of[e] (the expert cache) or e; the shared expert's
  // at sh_e (E, or the cache's slot count)
  const int32_t* slot_of;
  int sh_e;
  // the work split's divisors: stages per shared / routed unit in each phase, units per
  // expert in each phase
  FastDiv fd_s1, fd_s1q, fd_s2, fd_s2q, fd_u1, fd_u2;
};

// Shared memory: rings (codes, then scales), the phase-dependent area (phase 1: token as
// f16 [and, Q2 form, as e4m3 codes in 8-group order], its scales, stage partials;
// phase 2: up to three experts' h as f16 [Q2 form: the shared expert's as f16, two
// routed experts' as e4m3 codes in 8-group order], scales, stage partials), barriers,
// routing facts.  8-group order: each 8 consecutive codes as the 4 even then the 4 odd
// elements, the order of the 2-bit decode's e4m3 words.
struct DcSmem {
  int d, f;
  bool q2;
  static constexpr int kOffScales = kDcWarps * kDcStages * kDcCodeBytes;
  static constexpr int kOffArea = kOffScales + kDcWarps * kDcStages * kDcScaleBytes;
  __host__ __device__ int p1_q8() const { return kOffArea + 2 * d; }  // Q2 form
  __host__ __device__ int p1_bs() const { return kOffArea + (q2 ? 3 : 2) * d; }
  __host__ __device__ int p1_part() const { return p1_bs() + d / 32; }
  __host__ __device__ int p1_end() const { return p1_part() + kDcMaxUnits * (d / 512) * 64; }
  // phase 2: byte offset of local slot ls's activations
  __host__ __device__ int p2_act(int ls) const {
    return kOffArea + (q2 && ls > 0 ? 2 * f + (ls - 1) * f : ls * 2 * f);
  }
  __host__ __device__ int p2_bs() const { return kOffArea + (q2 ? 4 : 2 * kDcP2Slots) * f; }
  __host__ __device__ int p2_part() const { return p2_bs() + kDcP2Slots * (f / 32); }
  __host__ __device__ int p2_end() const { return p2_part() + kDcMaxUnits * (f / 512) * 64; }
  __host__ __device__ int bars() const {
    const int e = p1_end() > p2_end() ? p1_end() : p2_end();
    return (e + 7) / 8 * 8;
  }
  // ring barriers [warp][stage], the stall barrier
  __host__ __device__ int info() const { return bars() + (kDcWarps * kDcStages + 1) * 8; }
  // int words: abort, n_active, then per slot (expert, row0, rows), then per pair
  // (weight, pos)
  __host__ __device__ int bytes() const { return info() + 4 * (4 + 3 * kDcMaxSlots + 64) + 1024; }
};

__device__ __forceinline__ void ue8m0x4_f32(uint32_t w, float (&f)[4]) {
  const uint32_t m = 0x7F800000u, e0 = 0x00400000u;
  f[0] = __uint_as_float(max((w << 23) & m, e0));
  f[1] = __uint_as_float(max((w << 15) & m, e0));
  f[2] = __uint_as_float(max((w << 7) & m, e0));
  f[3] = __uint_as_float(max((w >> 1) & m, e0));
}

// Byte offset in a stage of bytes 4t..4t+3 of 32-block b (0..15) of stage row r (phase 1:
// rows 0-7 gate, 8-15 up, boxes [matrix][half][8 rows]; phase 2: boxes [half][16 rows]);
// the 128-byte swizzle XORs the 16-byte chunk with the row index mod 8.
template <int PH>
__device__ __forceinline__ uint32_t code_offset(int r, int b, int t) {
  const int half = b >> 3, chunk = b & 7;
  uint32_t box, rb;
  if (PH == 1) {
    box = (uint32_t)((r >> 3) * 2 + half) * 1024u;
    rb = (uint32_t)(r & 7);
  } else {
    box = (uint32_t)half * 2048u;
    rb = (uint32_t)r;
  }
  return box + rb * 128u + ((uint32_t)(chunk ^ (r & 7)) << 4) + 4u * (uint32_t)t;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}
__device__ __forceinline__ unsigned long long atom_add_acq_rel_u64(unsigned long long* p,
                                                                   unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v)
               : "memory");
  return old;
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// The bounded grid barrier (see g_grid_bar); false if the wait ran out.  ok_s: a word of
// shared memory that carries thread 0's result to the CTA.  The CTA barrier orders the
// CTA's writes before thread 0's arrival, an acq_rel atomic that releases them at GPU
// scope; the arrivals form one release sequence, so a waiter's acquire load that sees the
// last arrival's count orders its later reads after every arrival.
__device__ bool grid_barrier(long long limit, int* status, volatile int* ok_s) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned long long G = gridDim.x;
    const unsigned long long old = atom_add_acq_rel_u64(&g_grid_bar, 1ull);
    const unsigned long long target = (old / G + 1) * G;
    if (old + 1 != target) {
      const uint64_t t0 = ptx::globaltimer();
      while (ld_acquire_u64(&g_grid_bar) < target) {
        if ((long long)(ptx::globaltimer() - t0) > limit) {
          atomicOr(status, kStatusTimeout);
          ok = 0;
          break;
        }
      }
    }
    *ok_s = ok;
  }
  __syncthreads();
  return *ok_s != 0;
}

// Unit ul / chunk c of task `task` in a CTA range whose first ns units have S stages each
// (the shared expert's) and the rest Sq (the routed experts'); true for a routed unit.
__device__ __forceinline__ bool locate(int task, int ns, const FastDiv& S, const FastDiv& Sq,
                                       int& ul, int& c) {
  if (task < ns * (int)S.d) {
    ul = S.div(task);
    c = task - ul * (int)S.d;
    return false;
  }
  const int r = task - ns * (int)S.d;
  const int u = Sq.div(r);
  ul = ns + u;
  c = r - u * (int)Sq.d;
  return true;
}

// e4m3 bytes of the 2-bit values -1.5, -0.5, 0.5, 1.5 (byte i = code i), the table of the
// byte-permute decode
constexpr uint32_t kQ2Lut = 0x3C30B0BCu;

// One 128-element chunk of weight rows g and g + 8 (2-bit codes) against the token: lane
// (g, t) holds code bytes 8t..8t+7 of the chunk of both rows (wa, wb: codes 32t..32t+31,
// code i of a word in bits 2i..2i+1) and the token's e4m3 codes of elements 32t..32t+31 in
// 8-group order (x01: elements 32t..32t+15, x23: 32t+16..32t+31).  Masking a word with
// 0x33333333 leaves its even codes in the low 2 bits of its nibbles, the word shifted right
// by 2 its odd codes; a byte permute indexed by 4 such nibbles looks up 4 e4m3 bytes.  MMA
// m takes elements 32t + 8m .. 32t + 8m + 7 of every lane t, the even ones in k-slots
// 4t..4t+3 and the odd ones in 16+4t..16+4t+3 of both operands, so the four MMAs sum each
// of the 128 products once (fp32 accumulation in the tensor core).
__device__ __forceinline__ void q2_chunk_dot(uint2 wa, uint2 wb, uint4 x01, uint4 x23,
                                             float (&c)[4]) {
  const uint32_t ea0 = wa.x & 0x33333333u, oa0 = (wa.x >> 2) & 0x33333333u;
  const uint32_t ea1 = wa.y & 0x33333333u, oa1 = (wa.y >> 2) & 0x33333333u;
  const uint32_t eb0 = wb.x & 0x33333333u, ob0 = (wb.x >> 2) & 0x33333333u;
  const uint32_t eb1 = wb.y & 0x33333333u, ob1 = (wb.y >> 2) & 0x33333333u;
  auto lut = [](uint32_t sel) { return ptx::prmt(kQ2Lut, 0u, sel); };
  ptx::mma_m16n8k32_e4m3_zero(c, lut(ea0), lut(eb0), lut(oa0), lut(ob0), x01.x, x01.y);
  ptx::mma_m16n8k32_e4m3(c, lut(ea0 >> 16), lut(eb0 >> 16), lut(oa0 >> 16), lut(ob0 >> 16),
                         x01.z, x01.w);
  ptx::mma_m16n8k32_e4m3(c, lut(ea1), lut(eb1), lut(oa1), lut(ob1), x23.x, x23.y);
  ptx::mma_m16n8k32_e4m3(c, lut(ea1 >> 16), lut(eb1 >> 16), lut(oa1 >> 16), lut(ob1 >> 16),
                         x23.z, x23.w);
}

// DK, FK: 0 for the sizes of the launch, or d and f fixed at compile time (the decode
// sizes' instantiation, whose work-split and layout arithmetic folds to constants).
template <int MODE, int PL, bool RQ, int DK = 0, int FK = 0>
__global__ void __launch_bounds__(kDcThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  const int d = DK ? DK : p.d, f = FK ? FK : p.f, E = p.E, k = p.k;
  const DcSmem L{d, f, RQ};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = gridDim.x, b = blockIdx.x;

  uint16_t* bx = reinterpret_cast<uint16_t*>(smem + DcSmem::kOffArea);  // f16 activations
  uint8_t* bxq = smem + L.p1_q8();  // Q2 form: the token's e4m3 codes in 8-group order
  float* bs1 = reinterpret_cast<float*>(smem + L.p1_bs());
  float* part1 = reinterpret_cast<float*>(smem + L.p1_part());
  float* bs2 = reinterpret_cast<float*>(smem + L.p2_bs());
  float* part2 = reinterpret_cast<float*>(smem + L.p2_part());
  const uint32_t bars = ptx::smem_u32(smem + L.bars());
  const uint32_t stall_bar = bars + 8u * (kDcWarps * kDcStages);
  int* info = reinterpret_cast<int*>(smem + L.info());
  volatile int* abort_flag = info;
  int* n_active = info + 1;
  volatile int* barrier_ok = info + 2;
  int* slot_e = info + 4;                      // [slot] expert
  int* slot_row = slot_e + kDcMaxSlots;        // [slot] first output row
  int* slot_n = slot_row + kDcMaxSlots;        // [slot] rows (pairs) of the expert
  float* pair_w = reinterpret_cast<float*>(slot_n + kDcMaxSlots);  // [j] gate weight
  int* pair_pos = slot_n + kDcMaxSlots + 32;   // [j] sorted position

  auto full = [&](int s) { return bars + 8u * (uint32_t)(warp * kDcStages + s); };
  auto codes_at = [&](int s) { return smem + (warp * kDcStages + s) * kDcCodeBytes; };
  auto scales_at = [&](int s) {
    return smem + DcSmem::kOffScales + (warp * kDcStages + s) * kDcScaleBytes;
  };

  // the token's scores (warp 0, for the routing) and its first 4096 values (warps 1-8, for
  // the quantisation) are loaded first, so their latency overlaps the set-up below
  float sc_v[PL];
  uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
  if (MODE == kModeForward && warp == 0) load_scores<PL>(p.scores, E, lane, sc_v);
  if (warp >= 1 && warp <= 8 && (threadIdx.x - 32) * 16 < d) {
    xa = *reinterpret_cast<const uint4*>(p.x + (threadIdx.x - 32) * 16);
    xb = *reinterpret_cast<const uint4*>(p.x + (threadIdx.x - 32) * 16 + 8);
  }
  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&p.tm_gc);
    ptx::prefetch_tmap(&p.tm_gs);
    ptx::prefetch_tmap(&p.tm_uc);
    ptx::prefetch_tmap(&p.tm_us);
    ptx::prefetch_tmap(&p.tm_dc);
    ptx::prefetch_tmap(&p.tm_ds);
    if (RQ) {
      ptx::prefetch_tmap(&p.tm_gq);
      ptx::prefetch_tmap(&p.tm_gqs);
      ptx::prefetch_tmap(&p.tm_uq);
      ptx::prefetch_tmap(&p.tm_uqs);
      ptx::prefetch_tmap(&p.tm_dq);
      ptx::prefetch_tmap(&p.tm_dqs);
    }
    *abort_flag = 0;
    ptx::mbar_init(stall_bar, 1);  // never arrived on: only the test stall waits on it
  }
  if (lane == 0)
    for (int s = 0; s < kDcStages; ++s) ptx::mbar_init(full(s), 1);
  ptx::fence_mbar_init();
  if (MODE == kModeForward && b == 0)  // combine counters start at zero (published by the
    for (int i = threadIdx.x; i < d / 16; i += kDcThreads) p.done2[i] = 0;  // grid barrier)
  __syncthreads();

  // stages per unit: shared (FP4, 512-element stages) and routed (FP4, or 2-bit with
  // 1024-element stages in the Q2 form)
  const int S1 = d / 512, S2 = f / 512;
  const int S1q = RQ ? d / 1024 : S1, S2q = RQ ? f / 1024 : S2;
  const int wsh = RQ ? 2 : 1;
  const int upe1 = f / 8, upe2 = d / 16;
  const FastDiv fd_s1 = DK ? FastDiv(DK / 512) : p.fd_s1;
  const FastDiv fd_s1q = DK ? FastDiv(RQ ? DK / 1024 : DK / 512) : p.fd_s1q;
  const FastDiv fd_s2 = FK ? FastDiv(FK / 512) : p.fd_s2;
  const FastDiv fd_s2q = FK ? FastDiv(RQ ? FK / 1024 : FK / 512) : p.fd_s2q;
  const FastDiv fd_u1 = FK ? FastDiv(FK / 8) : p.fd_u1;
  const FastDiv fd_u2 = DK ? FastDiv(DK / 16) : p.fd_u2;
  const uint64_t pol = ptx::make_policy_evict_first();

  // n_act routed experts (known after routing); ranges and task counts follow from it
  int n_act = MODE == kModeForward ? k : 0;
  Range r1(upe1, n_act, G, b, wsh), r2(upe2, n_act, G, b, wsh);
  int q1 = 0, q2 = 0;

  // copies of this warp's q-th stage (phase 1 while q < q1), issued by lane 0
  auto issue = [&](int q) {
    const int st = q % kDcStages;
    const uint32_t dc = ptx::smem_u32(codes_at(st)), ds = ptx::smem_u32(scales_at(st));
    ptx::mbar_arrive_expect_tx(full(st), kDcStageBytes);
    if (q < q1) {
      int ul, c;
      const bool routed = locate(warp + q * kDcWarps, r1.ns, fd_s1, fd_s1q, ul, c);
      int e, uin;
      if (!routed) {
        e = p.sh_e;
        uin = r1.s_lo + ul;
      } else {
        const int ru = r1.r_lo + ul - r1.ns;
        const int sl = fd_u1.div(ru);
        e = slot_e[sl];
        if (p.slot_of) e = p.slot_of[e];
        uin = ru - sl * upe1;
      }
      if (RQ && routed) {
        // 2-bit stage: 2 x 128 code bytes (1024 elements) per row; the 16-byte scale box
        // covers 2048 elements, of which this stage uses bytes 8(c % 2)..+8
        const int row = e * f + uin * 8;
        ptx::tma_load_3d_hint(dc, &p.tm_gq, 0, row, 2 * c, full(st), pol);
        ptx::tma_load_3d_hint(dc + 2048, &p.tm_uq, 0, row, 2 * c, full(st), pol);
        ptx::tma_load_2d_hint(ds, &p.tm_gqs, (c >> 1) * 16, row, full(st), pol);
        ptx::tma_load_2d_hint(ds + 128, &p.tm_uqs, (c >> 1) * 16, row, full(st), pol);
      } else {
        const int row = e * f + uin * 8;
        ptx::tma_load_3d_hint(dc, &p.tm_gc, 0, row, 2 * c, full(st), pol);
        ptx::tma_load_3d_hint(dc + 2048, &p.tm_uc, 0, row, 2 * c, full(st), pol);
        ptx::tma_load_2d_hint(ds, &p.tm_gs, c * 16, row, full(st), pol);
        ptx::tma_load_2d_hint(ds + 128, &p.tm_us, c * 16, row, full(st), pol);
      }
    } else {
      int ul, c;
      const bool routed = locate(warp + (q - q1) * kDcWarps, r2.ns, fd_s2, fd_s2q, ul, c);
      int e, uin;
      if (!routed) {
        e = p.sh_e;
        uin = r2.s_lo + ul;
      } else {
        const int ru = r2.r_lo + ul - r2.ns;
        const int sl = fd_u2.div(ru);
        e = slot_e[sl];
        if (p.slot_of) e = p.slot_of[e];
        uin = ru - sl * upe2;
      }
      const int row = e * d + uin * 16;
      if (RQ && routed) {
        ptx::tma_load_3d_hint(dc, &p.tm_dq, 0, row, 2 * c, full(st), pol);
        ptx::tma_load_2d_hint(ds, &p.tm_dqs, (c >> 1) * 16, row, full(st), pol);
      } else {
        ptx::tma_load_3d_hint(dc, &p.tm_dc, 0, row, 2 * c, full(st), pol);
        ptx::tma_load_2d_hint(ds, &p.tm_ds, c * 16, row, full(st), pol);
      }
    }
  };

  // the shared expert's first stages go out before routing is known
  int issued = 0;
  {
    q1 = r1.ns * S1 > warp ? (r1.ns * S1 - warp + kDcWarps - 1) / kDcWarps : 0;  // shared only
    const int early = q1 < kDcStages ? q1 : kDcStages;
    if (lane == 0)
      for (int q = 0; q < early; ++q) issue(q);
    issued = early;
  }

  // ---------------------------------------------------------------- routing / plan
  if (warp == 0) {
    if (MODE == kModeForward) {
      // top-k of the E scores and the gate weights; CTA 0 stores them with the dispatch
      route_token_warp<PL>(sc_v, E, k, lane, slot_e, slot_row, slot_n, pair_w, pair_pos,
                           b == 0 ? p.idx : nullptr, p.w, p.perm, p.pos);
      if (lane == 0) *n_active = k;
    } else {
      // active experts from the dispatch offsets, ascending: (expert, first row, rows)
      const int per = (E + 31) / 32;
      const int e0 = lane * per, e1 = min(E, e0 + per);
      int local = 0;
      for (int e = e0; e < e1; ++e) local += p.offsets_in[e + 1] > p.offsets_in[e] ? 1 : 0;
      int incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int tt = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += tt;
      }
      int i = incl - local;
      for (int e = e0; e < e1; ++e) {
        const int lo = p.offsets_in[e], hi = p.offsets_in[e + 1];
        if (hi > lo) {
          if (i < kDcMaxSlots - 1 && lo >= 0 && hi <= k) {
            slot_e[i] = e;
            slot_row[i] = lo;
            slot_n[i] = hi - lo;
          } else {
            atomicOr(p.status, kStatusBadIndex);
          }
          ++i;
        }
      }
      if (lane == 31) *n_active = incl < kDcMaxSlots - 1 ? incl : kDcMaxSlots - 1;
    }
  } else if (warp <= 8) {
    // the token: s = amax / 448 per 128-block (IEEE divide; 1 if amax = 0), q = e4m3(x / s)
    // rounded to nearest even; 8 threads per block, 16 values each; f16 copies in smem
    const int tid = threadIdx.x - 32;
    for (int c0 = tid * 16; c0 - (tid & 31) * 16 < d; c0 += 256 * 16) {
      const bool act = c0 < d;
      uint4 a = xa, bb = xb;  // the first round's values were loaded at the start
      if (act && c0 != tid * 16) {
        a = *reinterpret_cast<const uint4*>(p.x + c0);
        bb = *reinterpret_cast<const uint4*>(p.x + c0 + 8);
      }
      const float v[16] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                           bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w),
                           bf16_lo(bb.x), bf16_hi(bb.x), bf16_lo(bb.y), bf16_hi(bb.y),
                           bf16_lo(bb.z), bf16_hi(bb.z), bf16_lo(bb.w), bf16_hi(bb.w)};
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
      const float sc = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
      uint32_t packed[4], hx[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint16_t lo = ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i], sc), __fdiv_rn(v[4 * i + 1], sc));
        const uint16_t hi =
            ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i + 2], sc), __fdiv_rn(v[4 * i + 3], sc));
        packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
        hx[2 * i] = ptx::cvt_e4m3x2_f16x2(lo);
        hx[2 * i + 1] = ptx::cvt_e4m3x2_f16x2(hi);
      }
      if (act) {
        uint4* dst = reinterpret_cast<uint4*>(bx + c0);
        dst[0] = make_uint4(hx[0], hx[1], hx[2], hx[3]);
        dst[1] = make_uint4(hx[4], hx[5], hx[6], hx[7]);
        if ((tid & 7) == 0) bs1[c0 / 128] = sc;
        if (RQ)  // the 16 codes in 8-group order: even then odd elements of each 8
          *reinterpret_cast<uint4*>(bxq + c0) =
              make_uint4(ptx::prmt(packed[0], packed[1], 0x6420u), ptx::prmt(packed[0], packed[1], 0x7531u),
                         ptx::prmt(packed[2], packed[3], 0x6420u), ptx::prmt(packed[2], packed[3], 0x7531u));
        if (b == 0) {
          *reinterpret_cast<uint4*>(p.qx + c0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          if ((tid & 7) == 0) p.sx[c0 / 128] = sc;
        }
      }
    }
  }
  __syncthreads();

  n_act = *n_active;
  r1 = Range(upe1, n_act, G, b, wsh);
  r2 = Range(upe2, n_act, G, b, wsh);
  const int nt1 = r1.ns * S1 + r1.nr * S1q, nt2 = r2.ns * S2 + r2.nr * S2q;
  q1 = nt1 > warp ? (nt1 - warp + kDcWarps - 1) / kDcWarps : 0;
  q2 = nt2 > warp ? (nt2 - warp + kDcWarps - 1) / kDcWarps : 0;
  // the host keeps every range within these limits; a plan that breaks them stops here
  if (r1.nr < 0 || r2.nr < 0 || r1.units() > kDcMaxUnits || r2.units() > kDcMaxUnits ||
      r2.nr > r2.upe + 1) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusBadIndex);
    *abort_flag = 1;
  }
  const int qt = q1 + q2;
  if (!*abort_flag) {
    if (lane == 0)
      for (int q = issued; q < kDcStages && q < qt; ++q) issue(q);
    issued = max(issued, min(kDcStages, qt));
  }

  // CTA 0 stores the dispatch of the token (forward)
  if (MODE == kModeForward && b == 0) {
    for (int e = threadIdx.x; e <= E; e += kDcThreads) {
      int below = 0, hit = 0;
      for (int s = 0; s < k; ++s) {
        below += slot_e[s] < e ? 1 : 0;
        hit += slot_e[s] == e ? 1 : 0;
      }
      p.offsets[e] = below;
      if (e < E) p.counts[e] = hit;
    }
  }

  // phase 2's experts held by this CTA: local slot 0 = shared, 1.. = routed slots
  const int r2_slot0 = r2.r_lo / upe2;
  auto p2_local = [&](int ul, int& e, int& uin, int& ls, int& slot) {
    if (ul < r2.ns) {
      e = E;
      uin = r2.s_lo + ul;
      ls = 0;
      slot = n_act;
    } else {
      const int ru = r2.r_lo + ul - r2.ns;
      slot = fd_u2.div(ru);
      e = slot_e[slot];
      uin = ru - slot * upe2;
      ls = 1 + slot - r2_slot0;
    }
  };

  // ---------------------------------------------------------------- phases 1 and 2
  const int r0 = g, rr1 = g + 8;
  // the lane's 8 swizzled code offsets within a 128-byte row group: 16-byte chunk c of rows
  // g and g + 8 (both g mod 8) lies at ((c ^ g) << 4), plus 4t for the lane's 4 bytes; the
  // box and half offsets are compile-time constants (see code_offset)
  uint32_t off8[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) off8[c] = (uint32_t)g * 128u + ((uint32_t)(c ^ g) << 4) + 4u * t;
  const bool ok = !*abort_flag;
  int q = 0;

  // all warps arrive here once, after their phase-1 stages: h of this CTA's units to
  // the workspace, the grid barrier, then the h of phase 2's experts staged as f16
  auto phase_switch = [&]() {
    __syncthreads();
    if (!*abort_flag) {
      for (int i = threadIdx.x; i < r1.units() * 8; i += kDcThreads) {
        const int ul = i >> 3, r = i & 7;
        float gg = 0.f, uu = 0.f;
        const int Su = ul < r1.ns ? S1 : S1q;
        for (int c = 0; c < Su; ++c) {
          gg += part1[(ul * S1 + c) * kDcRows + r];
          uu += part1[(ul * S1 + c) * kDcRows + 8 + r];
        }
        int slot, uin;
        if (ul < r1.ns) {
          slot = n_act;
          uin = r1.s_lo + ul;
        } else {
          const int ru = r1.r_lo + ul - r1.ns;
          slot = fd_u1.div(ru);
          uin = ru - slot * upe1;
        }
        const float h = __fdividef(gg, 1.0f + expf(-gg)) * uu;
        p.hbuf[(size_t)slot * f + uin * 8 + r] = h;
      }
    }
    if (!grid_barrier(p.wait_ns, p.status, barrier_ok)) *abort_flag = 1;
    // stage h: one warp per (local slot, 128-block), 4 values per lane; a warp loads the
    // h of up to four of its tasks before quantising any, so their L2 latencies overlap
    const int nb = f / 128;
    const int nls = 1 + (r2.nr > 0 ? (r2.r_lo + r2.nr - 1) / upe2 - r2_slot0 + 1 : 0);
    if (!*abort_flag) {
      for (int w0 = warp; w0 < nls * nb; w0 += 4 * kDcWarps) {
        float4 hv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int wi = w0 + u * kDcWarps;
          const int ls = wi / nb, j = wi % nb;
          hv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (wi < nls * nb && !(ls == 0 && r2.ns == 0)) {
            const int slot = ls == 0 ? n_act : r2_slot0 + ls - 1;
            hv[u] = __ldcg(reinterpret_cast<const float4*>(p.hbuf + (size_t)slot * f + 128 * j +
                                                           4 * lane));
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int wi = w0 + u * kDcWarps;
          const int ls = wi / nb, j = wi % nb;
          if (wi >= nls * nb || (ls == 0 && r2.ns == 0)) continue;
          const int slot = ls == 0 ? n_act : r2_slot0 + ls - 1;
          const float4 h = hv[u];
          float amax = fmaxf(fmaxf(fabsf(h.x), fabsf(h.y)), fmaxf(fabsf(h.z), fabsf(h.w)));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          const float sc = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
          const uint16_t q01 = ptx::cvt_e4m3x2(__fdiv_rn(h.x, sc), __fdiv_rn(h.y, sc));
          const uint16_t q23 = ptx::cvt_e4m3x2(__fdiv_rn(h.z, sc), __fdiv_rn(h.w, sc));
          const uint32_t qw = (uint32_t)q01 | ((uint32_t)q23 << 16);
          if (RQ && ls > 0) {
            // a 2-bit expert's h: codes in 8-group order; lanes 2m and 2m + 1 hold elements
            // 8m..8m+7, the even lane stores the even ones, the odd lane the odd ones
            const uint32_t qo = __shfl_xor_sync(0xffffffffu, qw, 1);
            *reinterpret_cast<uint32_t*>(smem + L.p2_act(ls) + 128 * j + 4 * lane) =
                (lane & 1) ? ptx::prmt(qo, qw, 0x7531u) : ptx::prmt(qw, qo, 0x6420u);
          } else {
            uint32_t* dst = reinterpret_cast<uint32_t*>(smem + L.p2_act(ls) + 2 * (128 * j + 4 * lane));
            dst[0] = ptx::cvt_e4m3x2_f16x2(q01);
            dst[1] = ptx::cvt_e4m3x2_f16x2(q23);
          }
          if (lane == 0) bs2[ls * nb + j] = sc;
          // the CTA holding the expert's first unit also stores its codes and scales
          const bool owner = ls == 0 ? r2.s_lo == 0 : slot * upe2 >= r2.r_lo;
          if (owner) {
            const int rows = ls == 0 ? 1 : slot_n[slot];
            const int row0 = ls == 0 ? k : slot_row[slot];
            for (int rr = 0; rr < rows; ++rr) {
              *reinterpret_cast<uint32_t*>(p.qh + (size_t)(row0 + rr) * f + 128 * j + 4 * lane) = qw;
              if (lane == 0) p.sh[(size_t)(row0 + rr) * nb + j] = sc;
            }
          }
        }
      }
    }
    __syncthreads();
  };

  // one phase's stages of this warp (PH: 1 = gate/up, 2 = down), from q up to q_end;
  // returns false if a wait ran out or another warp gave up
  auto run = [&](auto phc, int q_end) -> bool {
    constexpr int PH = decltype(phc)::value;
    for (; q < q_end; ++q) {
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) return false;  // another warp gave up
      const int st = q % kDcStages;
      if (p.stall && b == 0 && warp == 0 && q == 0 &&
          !wait_warp(stall_bar, 0, p.wait_ns, abort_flag, p.status))
        return false;
      if (!wait_warp(full(st), (uint32_t)(q / kDcStages) & 1u, p.wait_ns, abort_flag, p.status))
        return false;
      const uint8_t* cst = codes_at(st);
      const uint8_t* sst = scales_at(st);
      const int task = warp + (PH == 1 ? q : q - q1) * kDcWarps;
      int ul, c;
      const bool routed = PH == 1 ? locate(task, r1.ns, fd_s1, fd_s1q, ul, c)
                                  : locate(task, r2.ns, fd_s2, fd_s2q, ul, c);
      const uint16_t* xb = bx;
      const uint8_t* xq = bxq;
      const float* sxb = bs1;
      if (PH == 2) {
        int e, uin, ls, slot;
        p2_local(ul, e, uin, ls, slot);
        xb = reinterpret_cast<const uint16_t*>(smem + L.p2_act(ls));
        xq = smem + L.p2_act(ls);
        sxb = bs2 + ls * (f / 128);
      }
      float acc0 = 0.f, acc1 = 0.f;  // rows g and g+8 of the stage, column 0 (the token)
      if (RQ && routed) {
        // 2-bit stage: 16 rows x 1024 elements, 8 chunks of 128; this stage's 8 scale bytes
        // of each row are bytes 8(c % 2)..8(c % 2)+7 of its 16-byte scale box row
        const uint2 sa = *reinterpret_cast<const uint2*>(sst + r0 * 16 + 8 * (c & 1));
        const uint2 sb = *reinterpret_cast<const uint2*>(sst + rr1 * 16 + 8 * (c & 1));
#pragma unroll 2
        for (int jj = 0; jj < 8; ++jj) {
          const int j = 8 * c + jj;  // the token's 128-block
          // the lane's 8 code bytes of chunk jj (16-byte chunks 2 (jj % 4), 2 (jj % 4) + 1
          // of the rows' 128-byte piece jj / 4): bytes 8t..8t+7, in 16-byte chunk
          // 2 (jj % 4) + t / 2 (swizzled with the row index mod 8) at byte 8 (t % 2)
          const uint32_t piece = (uint32_t)(jj >> 2);
          const uint32_t ba = PH == 1 ? piece * 1024u : piece * 2048u;
          const uint32_t bbx = PH == 1 ? 2048u + piece * 1024u : piece * 2048u + 1024u;
          const uint8_t* cp = cst + g * 128 + ((((2 * (jj & 3)) + (t >> 1)) ^ g) << 4) + 8 * (t & 1);
          const uint2 wa = *reinterpret_cast<const uint2*>(cp + ba);
          const uint2 wb = *reinterpret_cast<const uint2*>(cp + bbx);
          const uint4 x01 = *reinterpret_cast<const uint4*>(xq + 128 * j + 32 * t);
          const uint4 x23 = *reinterpret_cast<const uint4*>(xq + 128 * j + 32 * t + 16);
          float cq[4];
          q2_chunk_dot(wa, wb, x01, x23, cq);
          const uint32_t ea = ((jj < 4 ? sa.x : sa.y) >> (8 * (jj & 3))) & 0xFFu;
          const uint32_t eb = ((jj < 4 ? sb.x : sb.y) >> (8 * (jj & 3))) & 0xFFu;
          const float fa = __uint_as_float(max(ea << 23, 0x00400000u));  // 2^(e-127), exact
          const float fb = __uint_as_float(max(eb << 23, 0x00400000u));
          const float sxj = sxb[j];
          acc0 = fmaf(sxj, fa * cq[0], acc0);
          acc1 = fmaf(sxj, fb * cq[2], acc1);
        }
      } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = 4 * c + i;
        float fa[4], fb[4];
        ue8m0x4_f32(*reinterpret_cast<const uint32_t*>(sst + r0 * 16 + 4 * i), fa);
        ue8m0x4_f32(*reinterpret_cast<const uint32_t*>(sst + rr1 * 16 + 4 * i), fb);
        float pa = 0.f, pb = 0.f;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const int blk = 4 * i + bb;
          // rows g and g + 8: boxes [matrix][half][8 rows] (phase 1) or [half][16 rows]
          const uint32_t half = (uint32_t)(blk >> 3);
          const uint32_t ba = PH == 1 ? half * 1024u : half * 2048u;
          const uint32_t bbx = PH == 1 ? 2048u + half * 1024u : half * 2048u + 1024u;
          const uint8_t* cp = cst + off8[blk & 7];
          const uint32_t wa = *reinterpret_cast<const uint32_t*>(cp + ba);
          const uint32_t wb = *reinterpret_cast<const uint32_t*>(cp + bbx);
          uint32_t ha[4], hb[4];
          ptx::cvt_e2m1x8_f16(wa, ha);
          ptx::cvt_e2m1x8_f16(wb, hb);
          const uint4 xv = *reinterpret_cast<const uint4*>(xb + 128 * j + 32 * bb + 8 * t);
          float cb[4];
          ptx::mma_m16n8k16_f16_zero(cb, ha[0], hb[0], ha[1], hb[1], xv.x, xv.y);
          ptx::mma_m16n8k16_f16(cb, ha[2], hb[2], ha[3], hb[3], xv.z, xv.w);
          pa = fmaf(fa[bb], cb[0], pa);
          pb = fmaf(fb[bb], cb[2], pb);
        }
        const float sxj = sxb[j];
        acc0 = fmaf(sxj, pa, acc0);
        acc1 = fmaf(sxj, pb, acc1);
      }
      }
      __syncwarp();  // every lane is done with the stage: it may be refilled
      if (issued < qt) {
        if (lane == 0) issue(issued);
        ++issued;
      }
      if (t == 0) {
        float* pp = (PH == 1 ? part1 + (ul * S1 + c) * kDcRows : part2 + (ul * S2 + c) * kDcRows);
        pp[r0] = acc0;
        pp[rr1] = acc1;
      }
    }
    return true;
  };
  // let the copies this warp issued land before the CTA can go on or exit
  auto give_up = [&]() {
    *abort_flag = 1;
    if (lane == 0)
      for (int r = q; r < issued; ++r) drain_wait(full(r % kDcStages), (uint32_t)(r / kDcStages) & 1u);
    __syncwarp();
    q = issued;
  };

  if (!(ok && run(std::integral_constant<int, 1>(), q1))) give_up();
  phase_switch();
  if (!run(std::integral_constant<int, 2>(), qt)) give_up();
  __syncthreads();
  if (*abort_flag) return;

  // ---------------------------------------------------------------- phase-2 results
  for (int i = threadIdx.x; i < r2.units() * kDcRows; i += kDcThreads) {
    const int ul = i >> 4, r = i & 15;
    float y = 0.f;
    const int Su = ul < r2.ns ? S2 : S2q;
    for (int c = 0; c < Su; ++c) y += part2[(ul * S2 + c) * kDcRows + r];
    int e, uin, ls, slot;
    p2_local(ul, e, uin, ls, slot);
    const size_t m = (size_t)uin * 16 + r;
    if (ls == 0) {
      p.y_shared[m] = y;
    } else {
      for (int rr = 0; rr < slot_n[slot]; ++rr) p.y_routed[(size_t)(slot_row[slot] + rr) * d + m] = y;
    }
  }
  if (MODE == kModeForward) {
    // Per 16-row output block, the last of the k + 1 experts to finish it sums out.  The
    // CTA barrier orders the CTA's y writes before each warp's acq_rel count (a release at
    // GPU scope, as in grid_barrier); the count that finds n_act earlier arrivals acquires
    // every other expert's rows.  The k routed rows are loaded together, then summed in
    // j order.
    __syncthreads();
    for (int ul = warp; ul < r2.units(); ul += kDcWarps) {
      int e, uin, ls, slot;
      p2_local(ul, e, uin, ls, slot);
      int last = 0;
      if (lane == 0) last = atom_add_acq_rel(p.done2 + uin, 1) == n_act ? 1 : 0;
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last && lane < 16) {
        const size_t m = (size_t)uin * 16 + lane;
        float acc = __ldcg(p.y_shared + m);
        for (int j0 = 0; j0 < k; j0 += 8) {
          float yv[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            yv[jj] = j0 + jj < k ? __ldcg(p.y_routed + (size_t)pair_pos[j0 + jj] * d + m) : 0.f;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            if (j0 + jj < k) acc = fmaf(pair_w[j0 + jj], yv[jj], acc);
        }
        p.out[m] = acc;
      }
    }
  }
}


template <int MODE, int PL, bool RQ, int DK = 0, int FK = 0>
cudaError_t launch_one(const DecodeParams& prm, cudaStream_t s, int grid) {
  const DcSmem L{prm.d, prm.f, RQ};
  const size_t smem = (size_t)L.bytes();
  auto kern = decode_kernel<MODE, PL, RQ, DK, FK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barrier
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, prm);
}

}  // namespace

size_t decode_smem_bytes(int d, int f, bool q2) { return (size_t)DcSmem{d, f, q2}.bytes(); }

bool decode_fits(int k, int d, int f, int ctas, bool q2) {
  if (k < 1 || k > 32 || d % 512 || f % 512 || ctas < 1) return false;
  // 2-bit stages hold 1024 elements and read 16-byte scale boxes (2048 elements)
  if (q2 && (d % 2048 || f % 2048)) return false;
  const int upe1 = f / 8, upe2 = d / 16, wsh = q2 ? 2 : 1;
  // every CTA's ranges, for every count of active experts the kernel can meet: at most
  // kDcMaxUnits units per phase, a routed share that is not negative, and a phase-2 routed
  // range over at most two experts
  for (int n = 1; n <= k; ++n)
    for (int b = 0; b < ctas; ++b) {
      const Range r1(upe1, n, ctas, b, wsh), r2(upe2, n, ctas, b, wsh);
      if (r1.nr < 0 || r2.nr < 0 || r1.units() > kDcMaxUnits || r2.units() > kDcMaxUnits)
        return false;
      if (r2.nr > upe2 + 1) return false;
    }
  return true;
}

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t s, int num_sms) {
  if (a.forward && a.q2_gate_codes == nullptr && a.tc_ws != nullptr)
    return launch_decode_tc(a, s, num_sms);
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  const int maps_e = a.maps_E >= 0 ? a.maps_E : a.E;  // experts of the FP4 maps, shared last
  const long long rows1 = (long long)(maps_e + 1) * a.f, rows2 = (long long)(maps_e + 1) * a.d;
  if (!make_code_map(&p.tm_gc, a.gate_codes, a.d / 2, rows1, 8) ||
      !make_byte_map(&p.tm_gs, a.gate_scales, a.d / 32, rows1, 16, 8) ||
      !make_code_map(&p.tm_uc, a.up_codes, a.d / 2, rows1, 8) ||
      !make_byte_map(&p.tm_us, a.up_scales, a.d / 32, rows1, 16, 8) ||
      !make_code_map(&p.tm_dc, a.down_codes, a.f / 2, rows2, 16) ||
      !make_byte_map(&p.tm_ds, a.down_scales, a.f / 32, rows2, 16, 16))
    return cudaErrorInvalidValue;
  const bool q2 = a.q2_gate_codes != nullptr;
  if (q2) {  // the E routed experts in the 2-bit codec: codes [rows][K/4], scales [rows][K/128]
    const long long q1 = (long long)a.E * a.f, q2r = (long long)a.E * a.d;
    if (!make_code_map(&p.tm_gq, a.q2_gate_codes, a.d / 4, q1, 8) ||
        !make_byte_map(&p.tm_gqs, a.q2_gate_scales, a.d / 128, q1, 16, 8) ||
        !make_code_map(&p.tm_uq, a.q2_up_codes, a.d / 4, q1, 8) ||
        !make_byte_map(&p.tm_uqs, a.q2_up_scales, a.d / 128, q1, 16, 8) ||
        !make_code_map(&p.tm_dq, a.q2_down_codes, a.f / 4, q2r, 16) ||
        !make_byte_map(&p.tm_dqs, a.q2_down_scales, a.f / 128, q2r, 16, 16))
      return cudaErrorInvalidValue;
  }
  p.scores = a.scores;
  p.x = a.x;
  p.offsets_in = a.offsets_in;
  p.idx = a.idx;
  p.w = a.w_out;
  p.counts = a.counts;
  p.offsets = a.offsets;
  p.perm = a.perm;
  p.pos = a.pos;
  p.y_routed = a.y_routed;
  p.y_shared = a.y_shared;
  p.out = a.out;
  p.qx = a.qx;
  p.sx = a.sx;
  p.qh = a.qh;
  p.sh = a.sh;
  p.hbuf = a.hbuf;
  p.done2 = a.done2;
  p.E = a.E;
  p.k = a.k;
  p.d = a.d;
  p.f = a.f;
  p.wait_ns = a.wait_ns;
  p.status = a.status;
  p.stall = a.stall;
  p.slot_of = a.slot_of;
  p.sh_e = maps_e;
  // the kernel's S1, S1q, S2, S2q, upe1, upe2 (2-bit routed stages hold 1024 elements)
  p.fd_s1 = FastDiv((uint32_t)(a.d / 512));
  p.fd_s1q = FastDiv((uint32_t)(q2 ? a.d / 1024 : a.d / 512));
  p.fd_s2 = FastDiv((uint32_t)(a.f / 512));
  p.fd_s2q = FastDiv((uint32_t)(q2 ? a.f / 1024 : a.f / 512));
  p.fd_u1 = FastDiv((uint32_t)(a.f / 8));
  p.fd_u2 = FastDiv((uint32_t)(a.d / 16));
  const int grid = num_sms < kMaxCtas ? num_sms : kMaxCtas;
  const bool dec = a.d == 4096 && a.f == 2048;  // the decode sizes' instantiation
  if (q2) {  // forward only
    if (!a.forward) return cudaErrorInvalidValue;
    if (a.E <= 256 && dec) return launch_one<kModeForward, 8, true, 4096, 2048>(p, s, grid);
    if (a.E <= 256) return launch_one<kModeForward, 8, true>(p, s, grid);
    return launch_one<kModeForward, 32, true>(p, s, grid);
  }
  if (a.forward) {
    if (a.E <= 256 && dec) return launch_one<kModeForward, 8, false, 4096, 2048>(p, s, grid);
    if (a.E <= 256) return launch_one<kModeForward, 8, false>(p, s, grid);
    return launch_one<kModeForward, 32, false>(p, s, grid);
  }
  return launch_one<kModeFfn, 8, false>(p, s, grid);
}

cudaError_t reset_grid_barrier() {
  const unsigned long long zero = 0;
  return cudaMemcpyToSymbol(g_grid_bar, &zero, sizeof(zero));
}

}  // namespace bitmoe
