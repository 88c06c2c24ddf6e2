// Single-token decode of the whole MoE layer in one kernel, on the 5th-generation tensor
// cores: routing, dispatch, activation quantisation, gate/up FP4 GEMV, SwiGLU,
// re-quantisation, down FP4 GEMV and the routing-weighted combine.
//
// At T = 1 the layer is bound by reading the k + 1 selected experts' FP4 codes and block
// scales once (dpshk.com article, "核心实现三" and "核心实现四": an expert is read once,
// FP4 decoded inside the product; tcti.cn post, "DeepSeek-V4-Flash的可能性": decode is
// memory-bound).  The CUDA-core form of this kernel (decode.cu) decodes e2m1 to f16 in
// registers, and that integer work, not HBM, sets its pace.  Here no thread touches a
// weight: TMA unpacks the FP4 codes into byte containers in shared memory
// (CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B) and tcgen05.mma kind::mxf8f6f4.block_scale
// multiplies them with the token's e4m3 codes, applying the ue8m0 weight scales itself.
//
// One token against 128 weight rows is an M = 128, N = 8 product.  The token's fp32 block
// scales (amax / 448 per 128 elements) cannot ride in the MMA, so each 128-element K block
// j must keep its own sum: the B operand is block-diagonal.  K block j of B is an 8-row
// tile whose row (j / 2) mod 8 holds the token's 128 codes of block j and whose other rows
// are zero, so the block's products land in one accumulator column.  The even and odd K
// blocks (the two halves of a 256-wide stage) accumulate into two regions of 16 columns:
// two independent chains of MMAs, since an N = 8 MMA is short and a chain of them waits
// on its accumulator.  After the K range, column 16 cb + c' of a region holds the sum of
// K block 2 c' + cb, and the epilogue forms sum_j s_j * D[j] in fp32.  Phase 2 stages
// the e4m3 codes of h the same way, one block-diagonal tile set per expert.
//
// Work: a stage is one matrix's 128 rows x 256 K (16 KB of FP4 codes from HBM, 32 KB of
// containers in shared memory, 1 KB of scales).  A unit is one (128-row block, 256-wide K
// chunk): two stages (gate, up) in phase 1, one (down) in phase 2.  The units of each
// phase are split over the CTAs as in decode.cu (Range): every CTA first holds a share of
// the shared expert, whose stages stream before the routing is known.  A CTA's units of
// one (expert, row block) form a segment, accumulated in one of seven TMEM buffers; its
// partial row sums (a "piece") go to the workspace under the index of its first K chunk,
// with its length.  No atomics combine the pieces:
//   phase 1  each piece is published by a flag holding this launch's epoch (release); the
//            CTA holding a row block's first K chunk waits (bounded) for the others'
//            flags, adds the pieces in K order, and computes h = silu(g) * u for the
//            block's 128 h-rows and, as these are exactly one 128-element block of h, its
//            amax, scale and e4m3 codes;
//   barrier  a bounded grid barrier (all h codes written); the down weights stream into
//            the ring meanwhile;
//   phase 2  every CTA builds the block-diagonal tiles of its experts' h codes and writes
//            its down pieces;
//   barrier  a second grid barrier; then CTA b takes output rows [b d / G, (b+1) d / G):
//            each expert's y as its pieces' sum in K order, and out = y_shared +
//            sum_j w_j y_j in fixed j order.
// Results do not depend on timing.  A flag waits only on pieces that other CTAs write
// before any wait of theirs in the same order (pieces of later CTAs' first segments), so
// the waits cannot form a cycle.
//
// Warp roles (10 warps, one CTA per SM):
//   0     TMA producer: the stages' code boxes (evict-first L2 hint)
//   1     scale loader: the stages' ue8m0 bytes, gathered by cp.async into the
//         tcgen05.cp 32x128b.warpx4 layout (row m at byte (m%32)*16 + (m/32)*4)
//   2-3   MMA issuers: issuer h takes half h of every stage (the K block 2 kc + h), four
//         MMAs into its own accumulator columns; warp 2 also allocates TMEM
//   6-9   epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (weight row = lane); it
//         also runs the grid barriers, builds phase 2's B tiles and does the combine
// In the prologue warp 6 routes the token and warps 2-5 and 7-9 quantise it into the
// block-diagonal B tiles.
//
// Every wait is bounded (%globaltimer): an expired wait records MOE_ERR_TIMEOUT in the
// status word, the roles stop, the CTA still takes part in the grid barrier, lets its
// copies and MMAs land, frees TMEM and returns.
#include "internal.cuh"
#include "ptx.cuh"
#include "single_token.cuh"
#include "waits.cuh"

#include <cstring>

namespace bitmoe {

// Grid barrier of this kernel, one per device (zero when the module loads): the count of
// CTA arrivals, a multiple of G between barriers, as in decode.cu (the last arrival's add
// opens the barrier); it serves one launch at a time (every CTA holds a whole SM until all
// have passed it), and a launch passes it twice.  The count at entry also tags the
// workspace's piece flags: all CTAs read the same value (the previous launch on the stream
// has ended and this one's first barrier cannot open before every CTA has arrived), and it
// grows with every launch, so a flag an earlier launch left behind does not match.
__device__ unsigned long long g_tc_bar;

namespace {

constexpr int kTcStages = 5;                         // ring depth
constexpr int kTcIssuers = 2;                        // one per 128-K half of a stage
constexpr int kTcKs = 256;                           // K elements per stage
constexpr int kTcABlock = 128 * 128;                 // 128 rows x 128 containers
constexpr int kTcStageBytes = 2 * kTcABlock + 1024;  // two 128-K blocks + their scales
constexpr int kTcBufs = 7;                           // segment accumulator buffers
constexpr int kTcBufCols = 64;                       // [half][matrix][16 K chunks]
constexpr int kTcWarps = 10;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcEpi0 = 6;                           // first epilogue warp
constexpr int kTcMaxSlots = 33;                      // k <= 32 routed + the shared expert
constexpr int kTcP2Local = 3;                        // experts a CTA meets in phase 2
// TMEM columns: buffer b's accumulators at 64 b + 32 half + 16 matrix + K chunk; the
// issuers' weight scales at 448 + 4 half; B's scales (1.0) at 456
constexpr uint32_t kColSfa = kTcBufs * kTcBufCols;
constexpr uint32_t kColSfb = kColSfa + 4 * kTcIssuers;
static_assert(kColSfb + 4 <= 512, "TMEM columns");

struct TcParams {
  CUtensorMap tm_g, tm_u, tm_d;  // FP4 codes as 16U4 containers: box 128 K x 128 rows
  const uint8_t* gs;             // ue8m0 scales [rows][K/32]
  const uint8_t* us;
  const uint8_t* ds;
  const float* scores;           // [E] router scores
  const uint16_t* x;             // [d] bf16 token
  int32_t* idx;                  // outputs: [k], [k], [E], [E+1], [k], [k]
  float* w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* pos;
  float* y_routed;               // [k][d], row = pair's sorted position
  float* y_shared;               // [d]
  float* out;                    // [d]
  uint8_t* qx;                   // workspace: the token's codes [d], scales [d/128]
  float* sx;
  uint8_t* qh;                   // workspace: h codes [k+1][f], scales [k+1][f/128]
  float* sh;
  float* hbuf;                   // workspace: h [k+1][f] fp32 (shared last)
  float* part1;                  // workspace: phase-1 pieces [k+1][f/128][d/256][2][128]
  int* len1;                     //            their lengths [k+1][f/128][d/256]
  uint32_t* flag1;               //            their epochs (written last, release)
  float* part2;                  // workspace: phase-2 pieces [k+1][d/128][f/256][128]
  int* len2;                     //            their lengths [k+1][d/128][f/256]
  int E, k, d, f;
  long long wait_ns;
  int* status;
  int stall;  // test knob: CTA 0's producer first waits on a barrier nothing completes
  // weight rows: expert e's are at slot_of[e] (the expert cache) or e; the shared
  // expert's at sh_e
  const int32_t* slot_of;
  int sh_e;
};

// Shared memory (from a 1024-byte aligned base): the stage ring, the B tiles (phase 1: the
// token's d/128 tiles; phase 2: up to three experts' f/128 tiles each), B's scale bytes,
// barriers, then small arrays.
struct TcSmem {
  int d, f;
  __host__ __device__ int b_tiles() const {
    return d / 128 > kTcP2Local * (f / 128) ? d / 128 : kTcP2Local * (f / 128);
  }
  static constexpr int kOffB = kTcStages * kTcStageBytes;
  __host__ __device__ int sfb() const { return kOffB + b_tiles() * 1024; }
  __host__ __device__ int bars() const { return sfb() + 512; }
  // full, empty, scales-full per stage; acc-full, acc-empty per buffer; setup, phase-2 B
  // ready, drain per issuer, the test stall's (never completed)
  static constexpr int kNumBars = 3 * kTcStages + 2 * kTcBufs + 2 + kTcIssuers + 1;
  __host__ __device__ int info() const { return bars() + 8 * kNumBars; }
  // info words: tmem, abort, epoch, spare, barrier ok, piece mask, 2 spare; slot_e,
  // pair_pos, pair_w; a row block's piece lengths
  __host__ __device__ int sx() const { return info() + 4 * (8 + kTcMaxSlots + 64 + 16); }
  __host__ __device__ int shs() const { return sx() + 4 * (d / 128); }
  __host__ __device__ int red() const { return shs() + 4 * kTcP2Local * (f / 128); }
  __host__ __device__ int bytes() const { return red() + 16 + 1024; }  // + alignment slack
};

// One CTA's work: its units in both phases (Range, wsh = 1) and their coordinates, with
// the divisors of the per-stage arithmetic (units per expert, K chunks per row block).
struct TcPlan {
  Range r1, r2;
  int NK1, NK2, RB1, n1, n2;
  FastDiv fu1, fu2, fk1, fk2;
  __host__ __device__ TcPlan(int n_routed, int d, int f, int G, int b)
      : r1((f / 128) * (d / kTcKs), n_routed, G, b, 1),
        r2((d / 128) * (f / kTcKs), n_routed, G, b, 1),
        fu1((uint32_t)((f / 128) * (d / kTcKs))), fu2((uint32_t)((d / 128) * (f / kTcKs))),
        fk1((uint32_t)(d / kTcKs)), fk2((uint32_t)(f / kTcKs)) {
    NK1 = d / kTcKs;
    NK2 = f / kTcKs;
    RB1 = f / 128;
    n1 = 2 * r1.units();
    n2 = r2.units();
  }
};

// Unit ul of a phase's range (units per expert fu, K chunks per row block fk): slot (-1 =
// the shared expert), 128-row block, K chunk, and the first and last unit of its segment
// (the run of units of one expert and row block).
struct TcUnit {
  int slot, rb, kc, ua, ub;
};
__host__ __device__ inline TcUnit tc_unit(const Range& r, const FastDiv& fu, const FastDiv& fk,
                                          int ul) {
  TcUnit t;
  int u, lo, hi;
  const int NK = (int)fk.d;
  if (ul < r.ns) {
    t.slot = -1;
    u = r.s_lo + ul;
    lo = 0;
    hi = r.ns - 1;
  } else {
    const int ru = r.r_lo + ul - r.ns;
    t.slot = fu.div(ru);
    u = ru - t.slot * (int)fu.d;
    lo = r.ns;
    hi = r.units() - 1;
  }
  t.rb = fk.div(u);
  t.kc = u - t.rb * NK;
  t.ua = ul - t.kc > lo ? ul - t.kc : lo;
  t.ub = ul + (NK - 1 - t.kc) < hi ? ul + (NK - 1 - t.kc) : hi;
  return t;
}
// Segments of a phase's range (shared ones first).
__host__ __device__ inline int tc_segments(const Range& r, const FastDiv& fk) {
  const int a = r.ns > 0 ? fk.div(r.s_lo + r.ns - 1) - fk.div(r.s_lo) + 1 : 0;
  const int b = r.nr > 0 ? fk.div(r.r_lo + r.nr - 1) - fk.div(r.r_lo) + 1 : 0;
  return a + b;
}
// Index of unit ul's segment within its phase.
__host__ __device__ inline int tc_segment_of(const Range& r, const FastDiv& fk, int ul) {
  if (ul < r.ns) return fk.div(r.s_lo + ul) - fk.div(r.s_lo);
  const int a = r.ns > 0 ? fk.div(r.s_lo + r.ns - 1) - fk.div(r.s_lo) + 1 : 0;
  return a + fk.div(r.r_lo + ul - r.ns) - fk.div(r.r_lo);
}

// Stage q of the CTA (phase 1: q < n1, unit q / 2, matrix q % 2; phase 2: unit q - n1):
// its unit, phase, matrix, and the CTA-wide index of its segment.
struct TcStageInfo {
  TcUnit u;
  int ph, mat, seg, qa, qb;  // qa, qb: first and last stage of the segment
};
__host__ __device__ inline TcStageInfo tc_stage(const TcPlan& P, int q) {
  TcStageInfo s;
  if (q < P.n1) {
    s.ph = 1;
    s.mat = q & 1;
    s.u = tc_unit(P.r1, P.fu1, P.fk1, q >> 1);
    s.seg = tc_segment_of(P.r1, P.fk1, q >> 1);
    s.qa = 2 * s.u.ua;
    s.qb = 2 * s.u.ub + 1;
  } else {
    s.ph = 2;
    s.mat = 0;
    s.u = tc_unit(P.r2, P.fu2, P.fk2, q - P.n1);
    s.seg = tc_segments(P.r1, P.fk1) + tc_segment_of(P.r2, P.fk2, q - P.n1);
    s.qa = P.n1 + s.u.ua;
    s.qb = P.n1 + s.u.ub;
  }
  return s;
}

__device__ __forceinline__ void bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long atom_add_acq_rel_u64(unsigned long long* p,
                                                                   unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Ties the values of a tcgen05.ld to this point, so that no use of them is scheduled
// before the tcgen05.wait::ld that precedes it.
template <int N>
__device__ __forceinline__ void reg_fence(float (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}

// The bounded grid barrier, run by the 128 epilogue threads (et: 0..127); the other warps
// keep streaming.  The named barrier orders the group's writes before thread 0's
// acq_rel arrival, which releases them at GPU scope; the arrivals form one release
// sequence, so a waiter's acquire load that sees the last arrival's count orders its later
// reads after every arrival.
__device__ bool tc_grid_barrier(long long limit, int* status, volatile int* ok_s, int et) {
  bar_sync(1, 128);
  if (et == 0) {
    int ok = 1;
    const unsigned long long G = gridDim.x;
    const unsigned long long old = atom_add_acq_rel_u64(&g_tc_bar, 1ull);
    const unsigned long long target = (old / G + 1) * G;
    if (old + 1 != target) {
      const uint64_t t0 = ptx::globaltimer();
      while (ld_acquire_u64(&g_tc_bar) < target) {
        if ((long long)(ptx::globaltimer() - t0) > limit) {
          atomicOr(status, kStatusTimeout);
          ok = 0;
          break;
        }
      }
    }
    *ok_s = ok;
  }
  bar_sync(1, 128);
  return *ok_s != 0;
}

template <int PL>
__global__ void __launch_bounds__(kTcThreads, 1) decode_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  const TcSmem L{p.d, p.f};
  const int d = p.d, f = p.f, E = p.E, k = p.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const TcPlan P(k, d, f, (int)gridDim.x, b);
  const int nq = P.n1 + P.n2;
  const int nseg1 = tc_segments(P.r1, P.fk1);
  const int nb1 = d / 128, nb2 = f / 128;  // 128-element K blocks of each phase
  const int RB2 = d / 128;
  const int r2s0 = P.r2.r_lo / P.r2.upe;   // first routed slot of phase 2

  uint8_t* bt = smem + TcSmem::kOffB;  // B tiles
  const uint32_t bars = ptx::smem_u32(smem + L.bars());
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (kTcStages + s); };
  auto sfull = [&](int s) { return bars + 8u * (2 * kTcStages + s); };
  auto afull = [&](int buf) { return bars + 8u * (3 * kTcStages + buf); };
  auto aempty = [&](int buf) { return bars + 8u * (3 * kTcStages + kTcBufs + buf); };
  const uint32_t setup = bars + 8u * (3 * kTcStages + 2 * kTcBufs);
  const uint32_t b2rdy = setup + 8u;
  auto drain = [&](int i) { return setup + 16u + 8u * i; };
  const uint32_t stall_bar = drain(kTcIssuers);
  int* info = reinterpret_cast<int*>(smem + L.info());
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(info);
  volatile int* abort_flag = info + 1;
  volatile uint32_t* epoch_s = reinterpret_cast<volatile uint32_t*>(info + 2);
  volatile int* ok_s = info + 4;
  volatile int* smask = info + 5;
  int* slot_e = info + 8;
  int* pair_pos = slot_e + kTcMaxSlots;
  float* pair_w = reinterpret_cast<float*>(pair_pos + 32);
  int* lens = reinterpret_cast<int*>(pair_w + 32);  // [16]
  float* sxs = reinterpret_cast<float*>(smem + L.sx());
  float* shs = reinterpret_cast<float*>(smem + L.shs());
  float* red = reinterpret_cast<float*>(smem + L.red());

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&p.tm_g);
    ptx::prefetch_tmap(&p.tm_u);
    ptx::prefetch_tmap(&p.tm_d);
    for (int s = 0; s < kTcStages; ++s) {
      ptx::mbar_init(full(s), 1);    // TMA arrive.expect_tx (+ transaction bytes)
      ptx::mbar_init(empty(s), kTcIssuers);  // tcgen05.commit of both issuers
      ptx::mbar_init(sfull(s), 32);  // the scale loader's 32 cp.async arrivals
    }
    for (int buf = 0; buf < kTcBufs; ++buf) {
      ptx::mbar_init(afull(buf), kTcIssuers);  // both issuers' commits at a segment's end
      ptx::mbar_init(aempty(buf), 1);          // the epilogue has read the accumulators
    }
    ptx::mbar_init(setup, 1);
    ptx::mbar_init(b2rdy, 1);
    for (int i = 0; i < kTcIssuers; ++i) ptx::mbar_init(drain(i), 1);
    ptx::mbar_init(stall_bar, 1);  // never arrived on: only the test stall waits on it
    *abort_flag = 0;
    *epoch_s = (uint32_t)ld_acquire_u64(&g_tc_bar);
    ptx::fence_mbar_init();
  }
  if (warp == 2) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x < 128)  // B's scale bytes: all 1.0 (0x7F)
    reinterpret_cast<uint32_t*>(smem + L.sfb())[threadIdx.x] = 0x7F7F7F7Fu;
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t epoch = *epoch_s;

  // weight-row expert of a slot (-1: the shared expert), in the arrays' numbering
  auto expert_of = [&](int slot) {
    if (slot < 0) return p.sh_e;
    const int e = slot_e[slot];
    return p.slot_of ? (int)p.slot_of[e] : e;
  };
  const uint64_t pol = ptx::make_policy_evict_first();
  // stage q's two code boxes (128 rows x 128 K each, unpacked to byte containers)
  auto issue = [&](int q) {
    const TcStageInfo s = tc_stage(P, q);
    const int st = q % kTcStages;
    const uint32_t dst = ptx::smem_u32(smem + st * kTcStageBytes);
    const long long e = expert_of(s.u.slot);
    const CUtensorMap* m = s.ph == 2 ? &p.tm_d : (s.mat ? &p.tm_u : &p.tm_g);
    const int row = (int)(e * (s.ph == 1 ? f : d)) + s.u.rb * 128;
    ptx::mbar_arrive_expect_tx(full(st), 2u * 128u * 64u);  // packed FP4 bytes
    ptx::tma_load_2d_hint(dst, m, s.u.kc * kTcKs, row, full(st), pol);
    ptx::tma_load_2d_hint(dst + kTcABlock, m, s.u.kc * kTcKs + 128, row, full(st), pol);
  };
  // stage q's ue8m0 bytes: for each 128-K block, 4 per row, in the tcgen05.cp
  // 32x128b.warpx4 layout (row m at byte (m%32)*16 + (m/32)*4); all 32 lanes
  auto load_sf = [&](int q) {
    const TcStageInfo s = tc_stage(P, q);
    const int st = q % kTcStages;
    const uint32_t sf0 = ptx::smem_u32(smem + st * kTcStageBytes + 2 * kTcABlock);
    const long long e = expert_of(s.u.slot);
    const uint8_t* src = s.ph == 2 ? p.ds : (s.mat ? p.us : p.gs);
    const size_t ld = (size_t)(s.ph == 1 ? d : f) / 32;
    const size_t row0 = (size_t)(e * (s.ph == 1 ? f : d)) + (size_t)s.u.rb * 128;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb)
#pragma unroll
      for (int m1 = 0; m1 < 4; ++m1)
        ptx::cp_async_4(sf0 + cb * 512 + lane * 16 + m1 * 4,
                        src + (row0 + m1 * 32 + lane) * ld + s.u.kc * 8 + cb * 4);
    ptx::cp_async_arrive_noinc(sfull(st));
  };

  // ---------------------------------------------------------------- prologue
  // The shared expert's first stages go out before the routing is known; warp 6 routes
  // the token while warps 2-5 and 7-9 quantise it into the block-diagonal B tiles.
  const int early = 2 * P.r1.ns < kTcStages ? 2 * P.r1.ns : kTcStages;
  bool stalled = false;  // warp 0, lane 0: the test stall ran out (nothing was issued)
  if (warp == 0) {
    if (lane == 0) {
      stalled = p.stall && b == 0 && !wait_one(stall_bar, 0, p.wait_ns, abort_flag, p.status);
      if (!stalled)
        for (int q = 0; q < early; ++q) issue(q);
    }
  } else if (warp == 1) {
    for (int q = 0; q < early; ++q) load_sf(q);
  } else if (warp == kTcEpi0) {
    route_token_warp<PL>(p.scores, E, k, lane, slot_e, nullptr, nullptr, pair_w, pair_pos,
                         b == 0 ? p.idx : nullptr, p.w, p.perm, p.pos);
  } else {
    // s = amax / 448 per 128-block (IEEE divide; 1 if amax = 0), q = e4m3(x / s) rounded
    // to nearest even; 8 lanes per block, 16 values each.  Code block j goes to row j % 8
    // of B tile j (128-byte swizzle: 16-byte chunk c of row r at r*128 + (c ^ r)*16).
    const int qi = warp < kTcEpi0 ? warp - 2 : warp - 3;  // 0..6
    for (int base = qi * 512; base < d; base += 7 * 512) {
      const int c0 = base + lane * 16;
      const bool act = c0 < d;
      uint4 a = make_uint4(0, 0, 0, 0), bb = make_uint4(0, 0, 0, 0);
      if (act) {
        a = *reinterpret_cast<const uint4*>(p.x + c0);
        bb = *reinterpret_cast<const uint4*>(p.x + c0 + 8);
      }
      const uint32_t wv[8] = {a.x, a.y, a.z, a.w, bb.x, bb.y, bb.z, bb.w};
      float v[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(wv[i] << 16);
        v[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
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
        const uint16_t hi = ptx::cvt_e4m3x2(__fdiv_rn(v[4 * i + 2], sc), __fdiv_rn(v[4 * i + 3], sc));
        packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
      }
      if (act) {
        const int j = c0 >> 7, c = (c0 & 127) >> 4, r = (j >> 1) & 7;
        *reinterpret_cast<uint4*>(bt + j * 1024 + r * 128 + ((c ^ r) << 4)) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
        if ((lane & 7) == 0) sxs[j] = sc;
        if (b == 0) {
          *reinterpret_cast<uint4*>(p.qx + c0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          if ((lane & 7) == 0) p.sx[j] = sc;
        }
      }
    }
    // the other seven rows of every tile (those of phase 2 too) are zero
    for (int i = qi * 32 + lane; i < L.b_tiles() * 64; i += 7 * 32) {
      const int j = i >> 6, r = (i >> 3) & 7, c = i & 7;
      if (r != ((j >> 1) & 7)) *reinterpret_cast<uint4*>(bt + j * 1024 + r * 128 + (c << 4)) = make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_smem();  // the tiles are read by the tensor cores (async proxy)
  }
  __syncthreads();

  // ---------------------------------------------------------------- roles
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int q = stalled ? 0 : early;  // the next stage to issue
      bool ok = !stalled;
      for (; ok && q < nq; ++q) {
        const int st = q % kTcStages;
        if (*abort_flag ||
            !wait_one(empty(st), ((uint32_t)(q / kTcStages) & 1u) ^ 1u, p.wait_ns, abort_flag, p.status)) {
          ok = false;
          break;
        }
        issue(q);
      }
      // let every issued copy land before the CTA can exit (after an abort the issuers
      // may not have waited for the last ones)
      const int q0 = stalled ? 0 : (q - kTcStages < 0 ? 0 : q - kTcStages);
      for (int j = q0; j < q; ++j) drain_wait(full(j % kTcStages), (uint32_t)(j / kTcStages) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ scale loader
    for (int q = early; q < nq; ++q) {
      const int st = q % kTcStages;
      if (*abort_flag ||
          !wait_warp(empty(st), ((uint32_t)(q / kTcStages) & 1u) ^ 1u, p.wait_ns, abort_flag, p.status))
        break;
      load_sf(q);
    }
    ptx::cp_async_wait_all();  // no copy of this warp may still be in flight at exit
    __syncwarp();
  } else if (warp < kTcEpi0) {
    // ------------------------------------------------------------ MMA issuers
    // issuer hf (warps 2 and 3) takes half hf of every stage: K block 2 kc + hf into its
    // own accumulators (column kc of a 16-column region per matrix), so the two halves
    // form two independent chains of MMAs.  Warps 4 and 5 only help in the prologue.
    const int hf = warp - 2;
    if (hf < kTcIssuers && lane == 0) {
      bool ok = true;
      if (hf == 0) {  // B's scale factors into TMEM once; both issuers read them
        ptx::tc_cp_32x128b_x4(tmem + kColSfb, ptx::make_sdesc(ptx::smem_u32(smem + L.sfb()), 0, 128, 0));
        ptx::tc_commit(setup);
      } else {
        ok = wait_one(setup, 0, p.wait_ns, abort_flag, p.status);
        ptx::tc_fence_after();
      }
      // kind::mxf8f6f4 instruction descriptor: A = e2m1 (5), B = e4m3 (0), both K-major,
      // ue8m0 scales, N >> 3 at bit 17 (N = 8), M >> 4 at bit 24; A scale id at bits 29-30
      const uint32_t idesc0 = (5u << 7) | (0u << 10) | ((8u >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
      const uint32_t sfa = tmem + kColSfa + 4u * (uint32_t)hf;
      const uint32_t bt_u = ptx::smem_u32(bt);
      uint32_t touched = 0;  // (matrix, column group) pairs of the open segment written
      bool b2 = false;
      for (int q = 0; ok && q < nq; ++q) {
        const TcStageInfo s = tc_stage(P, q);
        const int st = q % kTcStages;
        const int buf = s.seg % kTcBufs;
        if (q == s.qa) {  // a segment's first stage: the epilogue must have read its buffer
          if (s.seg >= kTcBufs &&
              !wait_one(aempty(buf), (uint32_t)(s.seg / kTcBufs - 1) & 1u, p.wait_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          touched = 0;
        }
        if (s.ph == 2 && !b2) {  // phase 2's B tiles are built after the grid barrier
          if (!wait_one(b2rdy, 0, p.wait_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          b2 = true;
        }
        const uint32_t ph = (uint32_t)(q / kTcStages) & 1u;
        if (!wait_one(full(st), ph, p.wait_ns, abort_flag, p.status) ||
            !wait_one(sfull(st), ph, p.wait_ns, abort_flag, p.status)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        ptx::fence_proxy_async_smem();  // scale bytes came through cp.async (generic proxy)
        const uint32_t a0 = ptx::smem_u32(smem + st * kTcStageBytes) + (uint32_t)(hf * kTcABlock);
        const uint32_t sf0 = ptx::smem_u32(smem + st * kTcStageBytes) + 2 * kTcABlock + 512u * (uint32_t)hf;
        ptx::tc_cp_32x128b_x4(sfa, ptx::make_sdesc(sf0, 0, 128, 0));
        const int j = 2 * s.u.kc + hf;  // the 128-element K block
        const int grp = s.u.kc >> 3;
        const int ls = s.u.slot < 0 ? 0 : 1 + s.u.slot - r2s0;
        const uint32_t btile = bt_u + (uint32_t)((s.ph == 1 ? j : ls * nb2 + j) * 1024);
        const uint32_t acc = tmem + (uint32_t)(buf * kTcBufCols + hf * 32 + s.mat * 16 + 8 * grp);
        const uint32_t tb = 1u << (2 * s.mat + grp);
        const uint64_t da = ptx::make_sdesc(a0, 16, 1024, 2);
        const uint64_t db = ptx::make_sdesc(btile, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // four K = 32 steps through the 128-byte rows
          ptx::tc_mma_mxf8f6f4(acc, da + 2 * kk, db + 2 * kk, idesc0 | ((uint32_t)kk << 29), sfa,
                               tmem + kColSfb, kk == 0 ? ((touched & tb) ? 1u : 0u) : 1u);
        touched |= tb;
        ptx::tc_commit(empty(st));
        if (q == s.qb) ptx::tc_commit(afull(buf));  // the segment's accumulators are done
      }
      ptx::tc_commit(drain(hf));  // every MMA / copy of this thread done before teardown
      drain_wait(drain(hf), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = (warp - kTcEpi0) * 32 + lane;  // 0..127
    const int quad = warp & 3;                    // TMEM lanes 32 quad .. +31
    const int r = quad * 32 + lane;               // weight row within the 128-row block
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);

    if (b == 0) {  // the dispatch of the token
      for (int e = et; e <= E; e += 128) {
        int below = 0, hit = 0;
        for (int s = 0; s < k; ++s) {
          below += slot_e[s] < e ? 1 : 0;
          hit += slot_e[s] == e ? 1 : 0;
        }
        p.offsets[e] = below;
        if (e < E) p.counts[e] = hit;
      }
    }

    // Row sums of segment seg (K chunks kca..kcb of one row block), nm matrices: each K
    // block's column times its activation scale, added in K-block order.  The buffer is
    // released as soon as its columns are in registers.  False if a wait ran out or
    // another role gave up.
    auto segment_sums = [&](int seg, int kca, int kcb, int nm, const float* scl, int nb,
                            float (&acc)[2]) -> bool {
      const int buf = seg % kTcBufs;
      if (et == 0) wait_one(afull(buf), (uint32_t)(seg / kTcBufs) & 1u, p.wait_ns, abort_flag, p.status);
      bar_sync(1, 128);
      if (*abort_flag) return false;
      ptx::tc_fence_after();
      float v[2][2][16];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int m = 0; m < 2; ++m)
          if (m < nm) ptx::tc_ld_32x32b_x16(tl + (uint32_t)(buf * kTcBufCols + h2 * 32 + m * 16), v[h2][m]);
      ptx::tc_wait_ld();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int m = 0; m < 2; ++m) reg_fence(v[h2][m]);
      ptx::tc_fence_before();
      bar_sync(1, 128);
      if (et == 0) ptx::mbar_arrive(aempty(buf));
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        acc[m] = 0.f;
#pragma unroll
        for (int kc = 0; kc < 16; ++kc)
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int j = 2 * kc + h2;
            if (m < nm && kc >= kca && kc <= kcb && j < nb) acc[m] = fmaf(scl[j], v[h2][m][kc], acc[m]);
          }
      }
      return true;
    };

    // h of one row block whose first K chunk this CTA holds: wait (bounded) until every
    // piece's flag carries this launch's epoch, then g and u are the pieces' sums in K
    // order, h = silu(g) u, and the block's scale and e4m3 codes.  False on a timeout.
    auto finish_h = [&](int sidx, int rb, size_t base) -> bool {
      uint64_t t0 = 0;
      uint32_t mk = 0;
      for (;;) {
        if (et < P.NK1) {
          const uint32_t fl = ld_acquire_u32(p.flag1 + base + et);
          lens[et] = fl == epoch ? __ldcg(p.len1 + base + et) : 0;
        }
        bar_sync(1, 128);
        if (et == 0) {
          uint32_t m2 = 0;
          bool done = true;
          for (int kc = 0; kc < P.NK1;) {
            const int len = lens[kc];
            if (len == 0) {  // that piece is not in yet
              done = false;
              break;
            }
            if (len < 0 || len > P.NK1 - kc) {
              atomicOr(p.status, kStatusBadIndex);
              *abort_flag = 1;
              break;
            }
            m2 |= 1u << kc;
            kc += len;
          }
          if (!done) {
            m2 = 0;
            if (t0 == 0) t0 = ptx::globaltimer();
            if ((long long)(ptx::globaltimer() - t0) > p.wait_ns) {
              atomicOr(p.status, kStatusTimeout);
              *abort_flag = 1;
            }
          }
          *smask = (int)m2;
        }
        bar_sync(1, 128);
        mk = (uint32_t)*smask;
        if (*abort_flag) return false;
        if (mk) break;
      }
      float gv[16], uv[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        gv[c] = 0.f;
        uv[c] = 0.f;
        if ((mk >> c) & 1u) {
          gv[c] = __ldcg(p.part1 + ((base + c) * 2) * 128 + r);
          uv[c] = __ldcg(p.part1 + ((base + c) * 2 + 1) * 128 + r);
        }
      }
      float g = 0.f, uu = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        g += gv[c];
        uu += uv[c];
      }
      const float h = __fdividef(g, 1.0f + expf(-g)) * uu;
      const uint32_t am = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(h)));
      if (lane == 0) red[warp - kTcEpi0] = __uint_as_float(am);
      bar_sync(1, 128);
      const float amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      const float sc = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
      const size_t m = (size_t)sidx * f + (size_t)rb * 128 + r;
      p.qh[m] = (uint8_t)(ptx::cvt_e4m3x2(__fdiv_rn(h, sc), 0.f) & 0xFFu);
      p.hbuf[m] = h;
      if (et == 0) p.sh[(size_t)sidx * nb2 + rb] = sc;
      bar_sync(1, 128);  // red and lens are read before the next finisher writes them
      return true;
    };

    bool ok = !*abort_flag;

    // ---- phase 1: each segment's partial sums go out with their length and, last, a flag
    // (release); the CTA holding a row block's first K chunk finishes its h
    for (int ul = 0; ok && ul < P.r1.units();) {
      const TcUnit u = tc_unit(P.r1, P.fu1, P.fk1, ul);
      const int seg = tc_segment_of(P.r1, P.fk1, ul);
      const int len = u.ub - u.ua + 1;
      float acc[2];
      if (!segment_sums(seg, u.kc, u.kc + len - 1, 2, sxs, nb1, acc)) {
        ok = false;
        break;
      }
      const int sidx = u.slot < 0 ? k : u.slot;
      const size_t base = ((size_t)sidx * P.RB1 + u.rb) * P.NK1;
      const size_t pb = base + u.kc;
      p.part1[(pb * 2) * 128 + r] = acc[0];
      p.part1[(pb * 2 + 1) * 128 + r] = acc[1];
      if (et == 0) p.len1[pb] = len;
      bar_sync(1, 128);  // every thread's values before the flag
      if (et == 0) st_release_u32(p.flag1 + pb, epoch);
      if (u.kc == 0 && !finish_h(sidx, u.rb, base)) {
        ok = false;
        break;
      }
      ul = u.ub + 1;
    }

    // ---- grid barrier: every h code written; then phase 2's B tiles
    if (!tc_grid_barrier(p.wait_ns, p.status, ok_s, et)) *abort_flag = 1;
    ok = ok && !*abort_flag;
    const int nls = P.r2.nr > 0 ? 2 + (P.r2.r_lo + P.r2.nr - 1) / P.r2.upe - r2s0 : 1;
    if (ok) {
      // local expert ls: 0 = the shared one, 1.. = routed slots r2s0..; its tile j
      // (smem tile t = ls * nb2 + j) holds h codes of block j in row (j / 2) % 8 (swizzled
      // as in phase 1); the prologue zeroed every row but (t / 2) % 8, which is cleared if
      // it differs
      const int nch = nls * nb2 * 8;
      for (int i0 = 0; i0 < nch; i0 += 4 * 128) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // four loads in flight before any store
          const int i = i0 + u * 128 + et;
          v[u] = make_uint4(0, 0, 0, 0);
          if (i < nch) {
            const int t = i >> 3, ls = t / nb2, j = t % nb2, c = i & 7;
            if (!(ls == 0 && P.r2.ns == 0)) {
              const int sidx = ls == 0 ? k : r2s0 + ls - 1;
              v[u] = __ldcg(reinterpret_cast<const uint4*>(p.qh + (size_t)sidx * f + 128 * j + 16 * c));
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * 128 + et;
          if (i < nch) {
            const int t = i >> 3, j = t % nb2, c = i & 7, rr = (j >> 1) & 7, r0 = (t >> 1) & 7;
            *reinterpret_cast<uint4*>(bt + t * 1024 + rr * 128 + ((c ^ rr) << 4)) = v[u];
            if (r0 != rr) *reinterpret_cast<uint4*>(bt + t * 1024 + r0 * 128 + (c << 4)) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      for (int i = et; i < nls * nb2; i += 128) {
        const int ls = i / nb2, j = i % nb2;
        shs[i] = (ls == 0 && P.r2.ns == 0) ? 0.f : __ldcg(p.sh + (size_t)(ls == 0 ? k : r2s0 + ls - 1) * nb2 + j);
      }
      ptx::fence_proxy_async_smem();
    }
    bar_sync(1, 128);
    if (et == 0) ptx::mbar_arrive(b2rdy);  // also on abort: no issuer waits for it then

    // ---- phase 2: each segment's partial sums and length
    for (int ul = 0; ok && ul < P.r2.units();) {
      const TcUnit u = tc_unit(P.r2, P.fu2, P.fk2, ul);
      const int seg = nseg1 + tc_segment_of(P.r2, P.fk2, ul);
      const int ls = u.slot < 0 ? 0 : 1 + u.slot - r2s0;
      const int len = u.ub - u.ua + 1;
      float acc[2];
      if (!segment_sums(seg, u.kc, u.kc + len - 1, 1, shs + ls * nb2, nb2, acc)) {
        ok = false;
        break;
      }
      const int sidx = u.slot < 0 ? k : u.slot;
      const size_t pb = ((size_t)sidx * RB2 + u.rb) * P.NK2 + u.kc;
      p.part2[pb * 128 + r] = acc[0];
      if (et == 0) p.len2[pb] = len;
      ul = u.ub + 1;
    }

    // ---- grid barrier: every down piece written; then this CTA's share of the output
    // rows, [b d / G, (b + 1) d / G): y of every expert as its pieces' sum in K order, and
    // out = y_shared + sum_j w_j y_j in fixed j order
    if (!tc_grid_barrier(p.wait_ns, p.status, ok_s, et)) *abort_flag = 1;
    ok = ok && !*abort_flag;
    if (ok) {
      const int G = (int)gridDim.x;
      const int m0 = (int)((long long)b * d / G), m1 = (int)((long long)(b + 1) * d / G);
      const int nrows = m1 - m0, rbA = m0 / 128;
      const int nrb = nrows > 0 ? (m1 - 1) / 128 - rbA + 1 : 0;  // at most two
      const int S = k + 1;
      int* lz = reinterpret_cast<int*>(bt);                         // [S][nrb][16] lengths
      uint32_t* mz = reinterpret_cast<uint32_t*>(lz + S * nrb * 16);  // [S][nrb] piece starts
      float* yz = reinterpret_cast<float*>(mz + S * nrb);            // [S][nrows] y
      for (int i = et; i < S * nrb * P.NK2; i += 128) {
        const int sidx = i / (nrb * P.NK2), rb = (i / P.NK2) % nrb, kc = i % P.NK2;
        lz[(sidx * nrb + rb) * 16 + kc] = __ldcg(p.len2 + ((size_t)sidx * RB2 + rbA + rb) * P.NK2 + kc);
      }
      bar_sync(1, 128);
      for (int i = et; i < S * nrb; i += 128) {
        uint32_t m2 = 0;
        for (int kc = 0; kc < P.NK2;) {
          const int len = lz[i * 16 + kc];
          if (len < 1 || len > P.NK2 - kc) {
            atomicOr(p.status, kStatusBadIndex);
            break;
          }
          m2 |= 1u << kc;
          kc += len;
        }
        mz[i] = m2;
      }
      bar_sync(1, 128);
      for (int i = et; i < S * nrows; i += 128) {
        const int sidx = i / nrows, row = m0 + i % nrows, rb = row / 128 - rbA, rr = row % 128;
        const uint32_t mk = mz[sidx * nrb + rb];
        const size_t base = ((size_t)sidx * RB2 + rbA + rb) * P.NK2;
        float yv[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) yv[c] = ((mk >> c) & 1u) ? __ldcg(p.part2 + (base + c) * 128 + rr) : 0.f;
        float y = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) y += yv[c];
        yz[i] = y;
        if (sidx == k) p.y_shared[row] = y;
        else p.y_routed[(size_t)sidx * d + row] = y;
      }
      bar_sync(1, 128);
      for (int i = et; i < nrows; i += 128) {
        float o = yz[k * nrows + i];
        for (int j = 0; j < k; ++j) o = fmaf(pair_w[j], yz[pair_pos[j] * nrows + i], o);
        p.out[m0 + i] = o;
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
// 2-D map over FP4 codes [rows][K/2 bytes] that TMA unpacks into byte containers: box =
// 128 elements of K x 128 rows, 128-byte swizzle (the UMMA shared-memory descriptors'
// layout).
bool make_fp4_map(CUtensorMap* m, const void* base, int K, long long rows) {
  EncodeTiledFn fn = tensor_map_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  const cuuint32_t box[2] = {128u, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int PL>
cudaError_t launch_tc(const TcParams& prm, cudaStream_t s, int grid) {
  const size_t smem = (size_t)TcSmem{prm.d, prm.f}.bytes();
  auto kern = decode_tc_kernel<PL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barrier
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, prm);
}

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// Workspace of the kernel, in order: part1, len1, flag1, part2, len2.
struct TcWs {
  size_t part1, len1, flag1, part2, len2, total;
  TcWs(int k, int d, int f) {
    const size_t S = (size_t)k + 1, RB1 = f / 128, RB2 = d / 128, NK1 = d / kTcKs, NK2 = f / kTcKs;
    part1 = 0;
    len1 = align256(part1 + S * RB1 * NK1 * 256 * sizeof(float));
    flag1 = align256(len1 + S * RB1 * NK1 * sizeof(int));
    part2 = align256(flag1 + S * RB1 * NK1 * sizeof(uint32_t));
    len2 = align256(part2 + S * RB2 * NK2 * 128 * sizeof(float));
    total = align256(len2 + S * RB2 * NK2 * sizeof(int));
  }
};

}  // namespace

size_t decode_tc_ws_bytes(int k, int d, int f) { return TcWs(k, d, f).total; }

size_t decode_tc_smem_bytes(int d, int f) { return (size_t)TcSmem{d, f}.bytes(); }

bool decode_tc_fits(int k, int d, int f, int ctas) {
  // K chunks of 256; K <= 4096 (two column groups per accumulator region)
  if (k < 1 || k > 32 || ctas < 1 || d % kTcKs || f % kTcKs || d > 4096 || f > 4096) return false;
  if (decode_tc_smem_bytes(d, f) > 232448) return false;
  // every CTA's ranges: a routed share that is not negative, a phase-2 routed range over
  // at most two experts (the B tiles hold three experts' h), and the combine's rows
  const TcSmem L{d, f};
  for (int b = 0; b < ctas; ++b) {
    const TcPlan P(k, d, f, ctas, b);
    if (P.r1.nr < 0 || P.r2.nr < 0 || P.r2.nr > P.r2.upe + 1) return false;
    // the combine's rows: within two row blocks, its scratch within the B tiles' space
    const int m0 = (int)((long long)b * d / ctas), m1 = (int)((long long)(b + 1) * d / ctas);
    const int nrb = m1 > m0 ? (m1 - 1) / 128 - m0 / 128 + 1 : 0;
    if (nrb > 2 || (size_t)(k + 1) * (nrb * 17 + (m1 - m0)) * 4 > (size_t)L.b_tiles() * 1024)
      return false;
  }
  return true;
}

cudaError_t launch_decode_tc(const DecodeLaunch& a, cudaStream_t s, int num_sms) {
  TcParams p;
  memset(&p, 0, sizeof(p));
  const int maps_e = a.maps_E >= 0 ? a.maps_E : a.E;  // experts of the maps, shared last
  const long long rows1 = (long long)(maps_e + 1) * a.f, rows2 = (long long)(maps_e + 1) * a.d;
  if (!make_fp4_map(&p.tm_g, a.gate_codes, a.d, rows1) ||
      !make_fp4_map(&p.tm_u, a.up_codes, a.d, rows1) ||
      !make_fp4_map(&p.tm_d, a.down_codes, a.f, rows2))
    return cudaErrorInvalidValue;
  const TcWs W(a.k, a.d, a.f);
  p.gs = a.gate_scales;
  p.us = a.up_scales;
  p.ds = a.down_scales;
  p.scores = a.scores;
  p.x = a.x;
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
  p.part1 = reinterpret_cast<float*>(a.tc_ws + W.part1);
  p.len1 = reinterpret_cast<int*>(a.tc_ws + W.len1);
  p.flag1 = reinterpret_cast<uint32_t*>(a.tc_ws + W.flag1);
  p.part2 = reinterpret_cast<float*>(a.tc_ws + W.part2);
  p.len2 = reinterpret_cast<int*>(a.tc_ws + W.len2);
  p.E = a.E;
  p.k = a.k;
  p.d = a.d;
  p.f = a.f;
  p.wait_ns = a.wait_ns;
  p.status = a.status;
  p.stall = a.stall;
  p.slot_of = a.slot_of;
  p.sh_e = maps_e;
  const int grid = num_sms < kMaxCtas ? num_sms : kMaxCtas;
  if (a.E <= 256) return launch_tc<8>(p, s, grid);
  return launch_tc<32>(p, s, grid);
}

// After a timeout a CTA may have left the barrier mid-count: move the count to a multiple
// of the grid size (ctas) above it, with no arrival pending.  The count only grows, so the
// epoch tags of the piece flags stay unique.
cudaError_t reset_tc_barrier(int ctas) {
  unsigned long long v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_tc_bar, sizeof(v));
  if (e != cudaSuccess) return e;
  const unsigned long long G = ctas > 0 ? (unsigned long long)ctas : 1ull;
  v = (v / G + 2) * G;
  return cudaMemcpyToSymbol(g_tc_bar, &v, sizeof(v));
}

}  // namespace bitmoe
