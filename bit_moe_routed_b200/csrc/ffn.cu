// Expert FFN on the 5th-generation tensor cores: block-scaled FP4 (e2m1) weights x
// FP8 (e4m3) activations, tcgen05.mma kind::mxf8f6f4 with fp32 accumulators in TMEM.
//
// Pages followed: tcti.cn post, "补齐软件栈缺失" (fp4_gemm: FP8-quantised activation x
// FP4 packed weight; act_quant) and "DeepSeek-V4-Flash的可能性" (prefill compute-bound,
// decode memory-bound); dpshk.com article, "核心实现三" (an expert's weights are read
// once for every token routed to it) and "核心实现四" (FP4 dequantised inside the
// product, gate and up on one quantised input).  Here the dequantisation happens in
// the tensor core itself: TMA unpacks the FP4 codes into byte containers in shared
// memory and the MMA applies the ue8m0 block scales from TMEM.
//
// Tiles ("swap-AB"): a tile is (expert e, block of 128 or 256 weight rows, token tile of
// n <= NMAX rows).  The weight rows are the MMA's M (128 per MMA); the tokens are its N
// (n rounded up to 16), so ragged expert groups waste at most 15 columns.  Phase 1
// multiplies the gate AND up rows of the same 128 h-rows with one shared activation
// tile, then computes h = silu(g) * u and re-quantises it per 128-block to e4m3;
// phase 2 is the down projection writing fp32 y.
//
// Work split: the tiles' 128-wide K chunks are the unit.  Whole tiles go out in rounds
// (CTA b takes tiles b, b + G, b + 2G, ...), so the G CTAs always work on neighbouring
// tiles and the weight blocks of one expert share each activation chunk through L2.  The
// tiles left over after the last full round are cut into one run of chunks split evenly
// over the CTAs ("stream-K"), so every SM gets the same number of weight bytes whatever
// the number of tiles.  A tile cut between CTAs is finished by the CTA that completes its
// last segment: each writes its fp32 partial to a slot, the last one (an atomic count)
// adds the segments in fixed order, so results are deterministic.
//
// Activation scales are fp32 (amax/448), not ue8m0, so they cannot ride in the MMA:
// B's hardware scale is 1.0 and every K chunk is accumulated into a fresh TMEM partial
// that the epilogue warps fold into fp32 registers as acc += s * P.  A ring of NBUF
// TMEM partials lets the MMA run NBUF chunks ahead of the epilogue.
//
// L2: a layer's weights stream through once; the TMA loads mark them evict-first so the
// activation rows, which every weight block of an expert reads again, stay in L2.
//
// Warp roles (32 * (10 + issuers) threads, one CTA per SM, persistent):
//   warp 0   : TMA producer (weights, activations)
//   warp 1   : TMEM allocator; lane 0 issues tcgen05.cp / tcgen05.mma / commits for the
//              first (matrix, 128-row block) of a tile
//   warps 2-9: epilogue; warp w reads TMEM lanes 32*(w%4).., column half (w-2)/4
//   warp 10  : scale loader: the weights' ue8m0 bytes (cp.async gather into the
//              tcgen05.cp layout) and the tokens' fp32 activation scales of each chunk
//   warps 11+: lane 0 issues for each further (matrix, 128-row block): the up matrix in
//              phase 1, the second 128-row block of 256-row tiles
// Every wait is bounded by a %globaltimer limit; on expiry the kernel records a
// timeout in the status word, lets in-flight copies and MMAs land, frees TMEM and
// returns.
#include "internal.cuh"
#include "ptx.cuh"
#include "waits.cuh"

#include <cstring>
#include <mutex>

namespace bitmoe {
namespace {

constexpr int kEpiWarps = 8;
constexpr int kSfWarp = 2 + kEpiWarps;          // warp 10 loads the scales
constexpr int kIssuerWarp1 = kSfWarp + 1;       // warps 11.. issue MMAs beside warp 1
// One issuing thread per (matrix, 128-row block) of a tile: a thread issues at most one
// tcgen05.mma per ~120 cycles whatever its N, so small-N tiles need several issuers.
constexpr int ffn_issuers(int phase, int mr) { return (phase == 1 ? 2 : 1) * (mr / 128); }
constexpr int ffn_threads(int phase, int mr) { return 32 * (kIssuerWarp1 + ffn_issuers(phase, mr) - 1); }

struct FfnParams {
  CUtensorMap tmA0;  // gate (phase 1) / down (phase 2) codes, all experts stacked
  CUtensorMap tmA1;  // up codes (phase 1)
  CUtensorMap tmB;   // activation rows [R][K] e4m3
  const uint8_t* sfa0;
  const uint8_t* sfa1;
  const float* b_scales;  // [R][K/128]
  const int32_t* plan;
  int E, K, rows_per_expert, R, P, f, d;
  uint8_t* qh;
  float* sh;
  float* y_routed;
  float* y_shared;
  int* counters;          // per tile, zero on entry, left zero on exit
  float* partials;        // [kMaxCtas][2][ncap][nmat][128]
  int ncap;
  int l2_hints;           // bit 0: weight boxes evict-first; bit 1: activation boxes evict-last
  long long wait_ns;
  int* status;
};

template <int PHASE, int NMAX, int STAGES, int NBUF, int MR>
struct Cfg {
  static constexpr int kNumA = PHASE == 1 ? 2 : 1;
  static constexpr int kRB = MR / 128;       // 128-row MMA blocks per weight tile
  static constexpr int kIssuers = ffn_issuers(PHASE, MR);
  static constexpr int kThreads = ffn_threads(PHASE, MR);
  static constexpr int kATile = MR * 128;    // MR rows x 128 FP4 in byte containers
  static constexpr int kBTile = NMAX * 128;
  static constexpr int kSF = 512 * kRB;      // per matrix: one 512-byte scale block per 128 rows
  static constexpr int kStageRaw = kNumA * kATile + kBTile + kNumA * kSF;
  static constexpr int kStage = (kStageRaw + 1023) / 1024 * 1024;
  // epilogue: with two 128-row blocks each group of four warps owns one block and all
  // columns; with one block the two groups split the columns
  static constexpr int kCols = kRB == 2 ? NMAX : NMAX / 2;
  static constexpr int kGroups = kCols / 8;            // 8-column TMEM loads per matrix
  static constexpr int kAccCols = kNumA * kRB * NMAX;  // per TMEM buffer
  static constexpr int kColSFA0 = NBUF * kAccCols;
  static constexpr int kColSFA1 = kColSFA0 + 4 * kRB;
  static constexpr int kColSFB = kColSFA0 + 4 * kRB * kNumA;
  static_assert(MR == 128 || MR == 256, "weight tile rows");
  static_assert(kColSFB + 4 <= 512, "TMEM columns");
  static_assert(NMAX % 16 == 0 && kCols % 8 == 0, "tile width");
  // shared memory after the stages
  static constexpr int kOffSFB = STAGES * kStage;
  static constexpr int kOffBars = kOffSFB + 512;
  static constexpr int kNumBars = 3 * STAGES + 3 * NBUF + kIssuers + 1;
  static constexpr int kOffMisc = (kOffBars + 8 * kNumBars + 15) / 16 * 16;  // tmem slot, abort, fix-up word
  static constexpr int kOffAmax = kOffMisc + 16;               // [2 groups][4 warps][kCols] column maxima
  static constexpr int kOffInv = kOffAmax + 2 * 4 * kCols * 4;  // [2 groups][kCols] 1/s
  static constexpr int kOffSx = kOffInv + 2 * kCols * 4;        // [NBUF][NMAX] activation scales
  static constexpr int kOffTT = kOffSx + NBUF * NMAX * 4;       // plan prefix, E+2 ints
  __host__ __device__ static size_t smem_bytes(int E) {
    return 1024 + (size_t)kOffTT + (size_t)(E + 2) * 4;
  }
};

__device__ __forceinline__ void bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// atomic add at GPU scope with acquire-release ordering
__device__ __forceinline__ int atom_add_acq_rel(int* ptr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
  return old;
}
// Ties the values of a tcgen05.ld to this point, so that no use of them is scheduled
// before the tcgen05.wait::ld that precedes it.
template <int N>
__device__ __forceinline__ void reg_fence(float (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}
// Tile i -> (expert, 128-row block, first activation row, rows).  Tiles of one expert
// are ordered (block, token tile) so consecutive tiles share weight rows in L2.
__device__ __forceinline__ void decode_tile(const int32_t* ttbase, const int32_t* tiles, int E,
                                            int HB, int i, int& e, int& blk, int& row0, int& n) {
  int lo = 0, hi = E;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ttbase[mid] * HB <= i) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int nt = ttbase[e + 1] - ttbase[e];
  const int local = i - ttbase[e] * HB;
  blk = local / nt;
  const int tt = ttbase[e] + local % nt;
  row0 = __ldg(tiles + 2 * tt);
  n = __ldg(tiles + 2 * tt + 1);
}

// Even partition of W chunks over G CTAs: CTA b takes [bW/G, (b+1)W/G).
struct Split {
  unsigned long long W;
  int G;
  __device__ __forceinline__ unsigned long long begin(int b) const {
    return (unsigned long long)b * W / (unsigned long long)G;
  }
  __device__ __forceinline__ int owner(unsigned long long c) const {  // CTA holding chunk c
    return (int)(((c + 1) * (unsigned long long)G - 1) / W);
  }
};

// Work split of T tiles over G CTAs.  The first Q*G tiles (Q = T / G) go out whole, round
// j giving tile b + j*G to CTA b: the G CTAs always work on G consecutive tiles, so the
// weight blocks of one expert, which read the same activation chunks, run side by side and
// share them through L2.  The last T - Q*G tiles (the tail) form one sequence of chunks
// split evenly over the G CTAs (stream-K); a tail tile cut between CTAs is finished by
// the last of them to complete its segment.
struct Sched {
  int Q, G, b, nk, base;          // base = Q*G, the first tail tile
  Split tail;                     // over the tail's chunks
  unsigned long long tbeg, tend;  // this CTA's tail chunks
  __device__ Sched(int total_tiles, int nk_, int G_, int b_) {
    G = G_;
    b = b_;
    nk = nk_;
    Q = total_tiles / G;
    base = Q * G;
    tail = Split{(unsigned long long)(total_tiles - base) * (unsigned long long)nk, G};
    tbeg = tail.begin(b);
    tend = tail.begin(b + 1);
  }
};
// Walks one CTA's segments in order: (tile, first chunk, end chunk) of each.
struct Cursor {
  int j;
  unsigned long long c;
  __device__ bool next(const Sched& s, int& tile, int& k0, int& k1) {
    if (j < s.Q) {
      tile = s.b + j * s.G;
      k0 = 0;
      k1 = s.nk;
      ++j;
      return true;
    }
    if (c < s.tend) {
      tile = s.base + (int)(c / s.nk);
      k0 = (int)(c % s.nk);
      k1 = (int)min((unsigned long long)s.nk, (unsigned long long)k0 + (s.tend - c));
      c += (unsigned long long)(k1 - k0);
      return true;
    }
    return false;
  }
};

template <int PHASE, int NMAX, int STAGES, int NBUF, int MR>
__global__ void __launch_bounds__(ffn_threads(PHASE, MR), 1) ffn_kernel(const __grid_constant__ FfnParams p) {
  using C = Cfg<PHASE, NMAX, STAGES, NBUF, MR>;
  constexpr int kMat = PHASE == 1 ? 2 : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* sfb = smem + C::kOffSFB;
  const uint32_t bars = ptx::smem_u32(smem + C::kOffBars);
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (STAGES + s); };
  auto sf_full = [&](int s) { return bars + 8u * (2 * STAGES + s); };
  auto tfull = [&](int b) { return bars + 8u * (3 * STAGES + b); };
  auto tempty = [&](int b) { return bars + 8u * (3 * STAGES + NBUF + b); };
  auto sx_full = [&](int b) { return bars + 8u * (3 * STAGES + 2 * NBUF + b); };
  // one drain barrier per MMA issuer; setup: the B scale copy has landed
  auto drain = [&](int i) { return bars + 8u * (3 * STAGES + 3 * NBUF + i); };
  const uint32_t setup = bars + 8u * (3 * STAGES + 3 * NBUF + C::kIssuers);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* fix_word = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);
  float* amax_s = reinterpret_cast<float*>(smem + C::kOffAmax);
  float* inv_s = reinterpret_cast<float*>(smem + C::kOffInv);
  float* sxb = reinterpret_cast<float*>(smem + C::kOffSx);
  int32_t* s_ttbase = reinterpret_cast<int32_t*>(smem + C::kOffTT);

  const int nk = p.K / 128;
  const int HB = p.rows_per_expert / MR;
  const int32_t* g_tiles = p.plan + p.E + 2;
  const int32_t* g_ttbase = s_ttbase;

  ptx::griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full(s), 1);      // TMA arrive.expect_tx (+ transaction bytes)
      ptx::mbar_init(sf_full(s), 32);  // the 32 scale-loader lanes' cp.async arrivals
      ptx::mbar_init(empty(s), C::kIssuers);  // tcgen05.commit of each MMA issuer
    }
    for (int b = 0; b < NBUF; ++b) {
      ptx::mbar_init(tfull(b), C::kIssuers);
      ptx::mbar_init(tempty(b), kEpiWarps);
      ptx::mbar_init(sx_full(b), 32);
    }
    for (int i = 0; i < C::kIssuers; ++i) ptx::mbar_init(drain(i), 1);
    ptx::mbar_init(setup, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + 128)  // B scale factors: all 1.0 (0x7F)
    reinterpret_cast<uint32_t*>(sfb)[threadIdx.x - 64] = 0x7F7F7F7Fu;
  // everything above overlaps the end of the previous launch on the stream; the plan,
  // the activation rows and their scales are written by it
  ptx::griddep_wait();
  for (int e = threadIdx.x; e < p.E + 2; e += C::kThreads) s_ttbase[e] = __ldg(p.plan + e);
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 1 && lane == 0) {  // B scale factors into TMEM once; both issuers read them
    ptx::tc_cp_32x128b_x4(tmem + C::kColSFB, ptx::make_sdesc(ptx::smem_u32(sfb), 0, 128, 0));
    ptx::tc_commit(setup);
  }
  const int total_tiles = g_ttbase[p.E + 1] * HB;
  const Sched sch(total_tiles, nk, (int)gridDim.x, (int)blockIdx.x);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&p.tmA0);
      if (PHASE == 1) ptx::prefetch_tmap(&p.tmA1);
      ptx::prefetch_tmap(&p.tmB);
    }
    // Weights are read once per layer and activations once per weight block: the weight
    // stream should not push the activation rows out of L2 between their reuses.
    const uint64_t pol_a = (p.l2_hints & 1) ? ptx::make_policy_evict_first() : ptx::make_policy_evict_normal();
    const uint64_t pol_b = (p.l2_hints & 2) ? ptx::make_policy_evict_last() : ptx::make_policy_evict_normal();
    int it = 0;
    bool ok = true;
    Cursor cur{0, sch.tbeg};
    int ti, k0, k1;
    while (ok && cur.next(sch, ti, k0, k1)) {
      int e, blk, row0, n;
      decode_tile(g_ttbase, g_tiles, p.E, HB, ti, e, blk, row0, n);
      const int rowA = e * p.rows_per_expert + blk * MR;
      const int nB = (n + 15) / 16;
      const uint32_t tx = (uint32_t)(C::kNumA * MR * 64 + nB * 2048);  // packed FP4 + e4m3 bytes
      for (int kc = k0; kc < k1; ++kc) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (!wait_warp(empty(s), ph ^ 1u, p.wait_ns, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const uint32_t st_u = ptx::smem_u32(smem + s * C::kStage);
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(full(s), tx);
          ptx::tma_load_2d_hint(st_u, &p.tmA0, kc * 128, rowA, full(s), pol_a);
          if (PHASE == 1)
            ptx::tma_load_2d_hint(st_u + C::kATile, &p.tmA1, kc * 128, rowA, full(s), pol_a);
          for (int j = 0; j < nB; ++j)
            ptx::tma_load_2d_hint(st_u + C::kNumA * C::kATile + j * 2048, &p.tmB, kc * 128,
                                  row0 + 16 * j, full(s), pol_b);
        }
        ++it;
      }
    }
    __syncwarp();
    if (lane == 0 && !ok)  // let every issued TMA copy land before the CTA can exit
      for (int j = it - STAGES < 0 ? 0 : it - STAGES; j < it; ++j)
        drain_wait(full(j % STAGES), (uint32_t)(j / STAGES) & 1u);
  } else if (warp == kSfWarp) {
    // ------------------------------------------------------------ scale loader
    // Per chunk: (1) the weights' ue8m0 bytes, 4 (4 K-blocks of 32) per weight row,
    // gathered with cp.async into the stage in the tcgen05.cp 32x128b.warpx4 layout (row m
    // at byte (m%32)*16 + (m/32)*4); (2) the tokens' fp32 activation scales of the chunk's
    // 128-block, into the ring slot of the chunk's TMEM buffer, for the epilogue.  Each
    // lane's copies arrive on the barrier by themselves when they land
    // (cp.async.mbarrier.arrive.noinc), so this warp never waits for its own loads.
    const size_t ldsf = (size_t)(p.K / 32);
    int it = 0, ch = 0;
    bool ok = true;
    Cursor cur{0, sch.tbeg};
    int ti, k0, k1;
    while (ok && cur.next(sch, ti, k0, k1)) {
      int e, blk, row0, n;
      decode_tile(g_ttbase, g_tiles, p.E, HB, ti, e, blk, row0, n);
      const int rowA = e * p.rows_per_expert + blk * MR;
      for (int kc = k0; kc < k1; ++kc) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (!wait_warp(empty(s), ph ^ 1u, p.wait_ns, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const uint32_t sf0 = ptx::smem_u32(smem + s * C::kStage) + C::kNumA * C::kATile + C::kBTile;
#pragma unroll
        for (int rb = 0; rb < C::kRB; ++rb) {
#pragma unroll
          for (int m1 = 0; m1 < 4; ++m1) {
            const size_t r = (size_t)(rowA + rb * 128 + m1 * 32 + lane);
            const uint32_t off = rb * 512 + lane * 16 + m1 * 4;
            ptx::cp_async_4(sf0 + off, p.sfa0 + r * ldsf + kc * 4);
            if (PHASE == 1) ptx::cp_async_4(sf0 + C::kSF + off, p.sfa1 + r * ldsf + kc * 4);
          }
        }
        ptx::cp_async_arrive_noinc(sf_full(s));
        ++it;
        const int b = ch % NBUF;
        const uint32_t tph = (uint32_t)(ch / NBUF) & 1u;
        if (!wait_warp(tempty(b), tph ^ 1u, p.wait_ns, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const uint32_t dst = ptx::smem_u32(sxb + b * NMAX);
        for (int cc = lane; cc < n; cc += 32)
          ptx::cp_async_4(dst + 4u * cc, p.b_scales + (size_t)(row0 + cc) * nk + kc);
        ptx::cp_async_arrive_noinc(sx_full(b));
        ++ch;
      }
    }
    ptx::cp_async_wait_all();  // no copy of this warp may still be in flight at exit
    __syncwarp();
  } else if (warp == 1 || (warp >= kIssuerWarp1 && warp - kIssuerWarp1 + 1 < C::kIssuers)) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer i (warp 1 for i = 0, warp 10 + i otherwise) owns matrix m = i / kRB (gate or
    // down 0, up 1) and 128-row block rb = i % kRB of every tile.  All wait for the same
    // stage and TMEM buffer and commit to both barriers, which count one arrival each.
    const int issuer = warp == 1 ? 0 : warp - kIssuerWarp1 + 1;
    const int m = issuer / C::kRB;
    const int rbi = issuer % C::kRB;
    if (lane == 0) {
      int it = 0, ch = 0;
      bool ok = true;
      if (issuer != 0) {  // the B scale copy was issued by warp 1
        ok = wait_one(setup, 0, p.wait_ns, abort_flag, p.status);
        ptx::tc_fence_after();
      }
      const uint32_t col_sfa = (m == 0 ? C::kColSFA0 : C::kColSFA1) + 4 * rbi;
      Cursor cur{0, sch.tbeg};
      int ti, k0, k1;
      while (ok && cur.next(sch, ti, k0, k1)) {
        int e, blk, row0, n;
        decode_tile(g_ttbase, g_tiles, p.E, HB, ti, e, blk, row0, n);
        const uint32_t N = (uint32_t)((n + 15) & ~15);
        // kind::mxf8f6f4 instruction descriptor: A = e2m1 (5), B = e4m3 (0), both K-major,
        // ue8m0 scales, N >> 3 at bit 17, M >> 4 at bit 24; A scale id at bits 29-30.
        const uint32_t idesc0 = (5u << 7) | (0u << 10) | ((N >> 3) << 17) | (1u << 23) |
                                ((128u >> 4) << 24);
        for (int kc = k0; kc < k1; ++kc) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          const int b = ch % NBUF;
          const uint32_t tph = (uint32_t)(ch / NBUF) & 1u;
          if (!wait_one(tempty(b), tph ^ 1u, p.wait_ns, abort_flag, p.status)) { ok = false; break; }
          ptx::tc_fence_after();
          if (!wait_one(full(s), ph, p.wait_ns, abort_flag, p.status)) { ok = false; break; }
          if (!wait_one(sf_full(s), ph, p.wait_ns, abort_flag, p.status)) { ok = false; break; }
          ptx::tc_fence_after();
          ptx::fence_proxy_async_smem();  // scale bytes came through cp.async (generic proxy)
          const uint32_t a0 = ptx::smem_u32(smem + s * C::kStage) + m * C::kATile + rbi * 16384;
          const uint32_t bb = ptx::smem_u32(smem + s * C::kStage) + C::kNumA * C::kATile;
          const uint32_t sf0 = bb + C::kBTile + m * C::kSF + rbi * 512;
          ptx::tc_cp_32x128b_x4(tmem + col_sfa, ptx::make_sdesc(sf0, 0, 128, 0));
          const uint64_t db = ptx::make_sdesc(bb, 16, 1024, 2);
          const uint64_t da = ptx::make_sdesc(a0, 16, 1024, 2);
          const uint32_t acc = tmem + (uint32_t)(b * C::kAccCols + (m * C::kRB + rbi) * NMAX);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // four K = 32 steps through the 128-byte rows
            // scale id kk selects byte kk of each SFA word: the scale of K-block kk
            const uint32_t idesc = idesc0 | ((uint32_t)kk << 29);
            ptx::tc_mma_mxf8f6f4(acc, da + 2 * kk, db + 2 * kk, idesc, tmem + col_sfa,
                                 tmem + C::kColSFB, kk > 0 ? 1u : 0u);
          }
          ptx::tc_commit(empty(s));
          ptx::tc_commit(tfull(b));
          ++it;
          ++ch;
        }
      }
      ptx::tc_commit(drain(issuer));  // every MMA / copy of this thread done before teardown
      drain_wait(drain(issuer), 0);
    }
    __syncwarp();
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int q = warp & 3;
    const int h = ew >> 2;                          // warp group 0/1
    const int rb = C::kRB == 2 ? h : 0;             // 128-row block of the weight tile
    const int col0 = C::kRB == 2 ? 0 : h * C::kCols;  // first column of this warp
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    const size_t slot_floats = (size_t)p.ncap * kMat * MR;
    int ch = 0;
    bool ok = true;
    Cursor cur{0, sch.tbeg};
    int ti, k0, k1;
    while (cur.next(sch, ti, k0, k1)) {
      int e, blk, row0, n;
      decode_tile(g_ttbase, g_tiles, p.E, HB, ti, e, blk, row0, n);
      // columns of this warp that hold tokens; the others are computed but never stored
      const int jn = n - col0 < 0 ? 0 : (n - col0 < C::kCols ? n - col0 : C::kCols);
      float acc0[C::kCols], acc1[C::kCols];
#pragma unroll
      for (int j = 0; j < C::kCols; ++j) {
        acc0[j] = 0.f;
        acc1[j] = 0.f;
      }
      for (int kc = k0; kc < k1; ++kc) {
        const int b = ch % NBUF;
        const uint32_t tph = (uint32_t)(ch / NBUF) & 1u;
        // one warp waits for the chunk's partial and scales, then releases the others
        // through a named barrier (eight warps spinning on one mbarrier would compete
        // with the TMA and the MMA for shared memory)
        if (ew == 0 && ok) {
          ok = wait_warp(tfull(b), tph, p.wait_ns, abort_flag, p.status);
          ok = ok && wait_warp(sx_full(b), tph, p.wait_ns, abort_flag, p.status);
        }
        bar_sync(4, kEpiWarps * 32);
        ok = ok && *abort_flag == 0;
        ptx::tc_fence_after();
        if (ok && jn > 0) {
          // acc += s * P, 8 columns of each matrix per TMEM round trip
          const uint32_t base = tl + (uint32_t)(b * C::kAccCols + rb * NMAX + col0);
          const float4* sc4 = reinterpret_cast<const float4*>(sxb + b * NMAX + col0);
          auto group = [&](int g) {
            float v0[8], v1[8];
            ptx::tc_ld_32x32b_x8(base + 8 * g, v0);
            if (PHASE == 1) ptx::tc_ld_32x32b_x8(base + C::kRB * NMAX + 8 * g, v1);
            const float4 sa = sc4[2 * g], sb = sc4[2 * g + 1];
            ptx::tc_wait_ld();
            reg_fence(v0);
            if (PHASE == 1) reg_fence(v1);
            const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              acc0[8 * g + j] = fmaf(sv[j], v0[j], acc0[8 * g + j]);
              if (PHASE == 1) acc1[8 * g + j] = fmaf(sv[j], v1[j], acc1[8 * g + j]);
            }
          };
          if (jn > C::kCols - 8) {  // every group holds tokens: straight-line code
#pragma unroll
            for (int g = 0; g < C::kGroups; ++g) group(g);
          } else {  // few tokens (decode): only the groups that hold some
#pragma unroll
            for (int g = 0; g < C::kGroups; ++g) {
              if (8 * g >= jn) break;
              group(g);
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(tempty(b));
        ++ch;
      }

      // ---- stream-K fix-up of a tail tile cut between CTAs.  The tile's segments belong
      // to the CTAs owning its chunks (CTAs with empty ranges own none): walk them in order.
      const Split& sp = sch.tail;
      const int tt = ti - sch.base;  // index among the tail tiles (< 0: a whole tile)
      const unsigned long long t0c = (unsigned long long)(tt < 0 ? 0 : tt) * nk;
      int nseg = 0;
      if (tt >= 0)
        for (unsigned long long cc = t0c; cc < t0c + nk;) {
          ++nseg;
          cc = sp.begin(sp.owner(cc) + 1);
        }
      bool finish = true;
      const size_t lane_off = (size_t)rb * 128 + q * 32 + lane;
      if (nseg > 1) {
        const int my_slot = 2 * blockIdx.x + ((int)(sch.tbeg / nk) == tt ? 0 : 1);
        float* mine = p.partials + (size_t)my_slot * slot_floats;
        if (ok) {
#pragma unroll
          for (int j = 0; j < C::kCols; ++j) {
            if (j < jn) {
              const size_t o = (size_t)(col0 + j) * kMat * MR + lane_off;
              mine[o] = acc0[j];
              if (PHASE == 1) mine[o + MR] = acc1[j];
            }
          }
        }
        // one acq_rel atomic (after the barrier) publishes every thread's partial and, for
        // the last arrival, makes the other CTAs' partials visible to the whole CTA
        bar_sync(1, kEpiWarps * 32);
        if (ew == 0 && lane == 0)
          *fix_word = *abort_flag ? -1 : atom_add_acq_rel(p.counters + ti, 1);
        bar_sync(1, kEpiWarps * 32);
        const int arrived = *fix_word;
        finish = arrived == nseg - 1;
        if (finish && jn <= 4 && nseg <= 4) {
          // few columns (decode): every segment's loads in flight at once, then summed in
          // chunk order
          float v[4][4][kMat];
          unsigned long long cs = t0c;
#pragma unroll
          for (int si = 0; si < 4; ++si) {
            const bool have = si < nseg;
            const int s = have ? sp.owner(cs) : 0;
            const int slot = 2 * s + ((int)(sp.begin(s) / nk) == tt ? 0 : 1);
            if (have) cs = sp.begin(s + 1);
            const float* src = p.partials + (size_t)slot * slot_floats;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int m = 0; m < kMat; ++m)
                v[si][j][m] = have && j < jn
                                  ? __ldcg(src + (size_t)(col0 + j) * kMat * MR + lane_off + m * MR)
                                  : 0.f;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float a0 = v[0][j][0], a1 = v[0][j][kMat - 1];
#pragma unroll
            for (int q2 = 1; q2 < 4; ++q2)
              if (q2 < nseg) {
                a0 += v[q2][j][0];
                a1 += v[q2][j][kMat - 1];
              }
            if (j < C::kCols) {
              acc0[j] = a0;
              if (PHASE == 1) acc1[j] = a1;
            }
          }
          if (ew == 0 && lane == 0) p.counters[ti] = 0;  // ready for the next launch
        } else if (finish) {
          // all segments, this CTA's included, from their slots in chunk order: the sum
          // does not depend on which CTA finishes last
          bool first_seg = true;
          for (unsigned long long cs = t0c; cs < t0c + nk;) {
            const int s = sp.owner(cs);
            cs = sp.begin(s + 1);
            const int slot = 2 * s + ((int)(sp.begin(s) / nk) == tt ? 0 : 1);
            const float* src = p.partials + (size_t)slot * slot_floats;
#pragma unroll
            for (int j = 0; j < C::kCols; ++j) {
              if (j < jn) {
                const size_t o = (size_t)(col0 + j) * kMat * MR + lane_off;
                const float v0 = __ldcg(src + o);
                acc0[j] = first_seg ? v0 : acc0[j] + v0;
                if (PHASE == 1) {
                  const float v1 = __ldcg(src + o + MR);
                  acc1[j] = first_seg ? v1 : acc1[j] + v1;
                }
              }
            }
            first_seg = false;
          }
          if (ew == 0 && lane == 0) p.counters[ti] = 0;  // ready for the next launch
        }
      }
      finish = finish && ok;
      const int js = finish ? jn : 0;   // columns this warp stores
      const int hb = blk * C::kRB + rb;  // 128-wide block of h (phase 1) / of y (phase 2)

      if (PHASE == 1) {
        // h = silu(g) * u in place of g, then per-column (token) e4m3 re-quantisation over
        // the 128 rows: column maxima per warp, combined by one thread per column, which
        // writes s and 1/s; every thread then encodes its 128-row slice of each column.
#pragma unroll
        for (int j = 0; j < C::kCols; ++j) {
          const float g = acc0[j];
          acc0[j] = __fdividef(g, 1.0f + expf(-g)) * acc1[j];
        }
        float* am = amax_s + (h * 4 + q) * C::kCols;
#pragma unroll
        for (int j = 0; j < C::kCols; ++j) {
          const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(acc0[j])));
          if (lane == 0) am[j] = __uint_as_float(m);
        }
        bar_sync(2 + h, 128);
        const int t = q * 32 + lane;
        if (t < js) {
          const float* a = amax_s + h * 4 * C::kCols + t;
          const float amax =
              fmaxf(fmaxf(a[0], a[C::kCols]), fmaxf(a[2 * C::kCols], a[3 * C::kCols]));
          const float s = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
          inv_s[h * C::kCols + t] = __frcp_rn(s);
          p.sh[(size_t)(row0 + col0 + t) * (p.f / 128) + hb] = s;
        }
        bar_sync(2 + h, 128);
        const float4* inv4 = reinterpret_cast<const float4*>(inv_s + h * C::kCols);
        uint8_t* dst = p.qh + (size_t)(row0 + col0) * p.f + hb * 128 + q * 32 + lane;
#pragma unroll
        for (int j = 0; j < C::kCols; j += 4) {
          if (j >= js) break;
          const float4 r = inv4[j / 4];
          const uint16_t c01 = ptx::cvt_e4m3x2(acc0[j] * r.x, acc0[j + 1] * r.y);
          const uint16_t c23 = ptx::cvt_e4m3x2(acc0[j + 2] * r.z, acc0[j + 3] * r.w);
          if (j < js) dst[(size_t)j * p.f] = (uint8_t)(c01 & 0xFF);
          if (j + 1 < js) dst[(size_t)(j + 1) * p.f] = (uint8_t)(c01 >> 8);
          if (j + 2 < js) dst[(size_t)(j + 2) * p.f] = (uint8_t)(c23 & 0xFF);
          if (j + 3 < js) dst[(size_t)(j + 3) * p.f] = (uint8_t)(c23 >> 8);
        }
      } else {
#pragma unroll
        for (int j = 0; j < C::kCols; ++j) {
          if (j < js) {
            const int row = row0 + col0 + j;
            float* dst = row < p.P ? p.y_routed + (size_t)row * p.d
                                   : p.y_shared + (size_t)(row - p.P) * p.d;
            dst[(size_t)hb * 128 + q * 32 + lane] = acc0[j];
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
// 2-D map over a row-major matrix [rows][K]; box = 128 elements of K x box_rows rows,
// 128-byte swizzle (the layout the UMMA shared-memory descriptors expect).
bool make_map(CUtensorMap* m, const void* base, bool fp4, int K, long long rows, int box_rows) {
  EncodeTiledFn fn = tensor_map_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(fp4 ? K / 2 : K)};
  const cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(m, fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                        2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int PHASE, int NMAX, int STAGES, int NBUF, int MR>
cudaError_t launch_one(const FfnParams& prm, cudaStream_t s, int grid, bool overlap) {
  using C = Cfg<PHASE, NMAX, STAGES, NBUF, MR>;
  const size_t smem = C::smem_bytes(prm.E);
  cudaError_t err = cudaFuncSetAttribute(ffn_kernel<PHASE, NMAX, STAGES, NBUF, MR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(ffn_kernel<PHASE, NMAX, STAGES, NBUF, MR>, dim3(grid), dim3(C::kThreads), smem, s,
                    overlap, prm);
}

// (PHASE, NMAX) -> pipeline stages, TMEM partial buffers, weight rows per tile.  Small
// batches take 256-row tiles: one TMA box then moves 16 KB of FP4, which streams HBM far
// better than 8 KB boxes; large batches keep 128-row tiles to leave TMEM for wide N.
#define BITMOE_FFN_VARIANTS(X)                  \
  X(1, kNmaxSmall, 3, 3, 256)                   \
  X(1, kNmaxSmall, 5, 6, 128)                   \
  X(1, kNmaxLarge, 4, 2, 128)                   \
  X(2, kNmaxSmall, 5, 6, 256)                   \
  X(2, kNmaxSmall, 8, 8, 128)                   \
  X(2, kNmaxLarge, 6, 4, 128)

int tile_rows(int nmax, int rows_per_expert) {
  return nmax == kNmaxSmall && rows_per_expert % 256 == 0 ? 256 : 128;
}

}  // namespace

size_t ffn_smem_bytes(int phase, int nmax, int E, int rows_per_expert) {
  const int mr = tile_rows(nmax, rows_per_expert);
#define X(P, N, S, B, M) \
  if (phase == P && nmax == N && mr == M) return Cfg<P, N, S, B, M>::smem_bytes(E);
  BITMOE_FFN_VARIANTS(X)
#undef X
  return 0;
}

cudaError_t launch_ffn(int phase, int nmax, const FfnArgs& a, cudaStream_t s, int num_sms) {
  FfnParams prm;
  memset(&prm, 0, sizeof(prm));
  const long long rows_total = (long long)(a.E + 1) * a.rows_per_expert;
  const int mr = tile_rows(nmax, a.rows_per_expert);
  if (!make_map(&prm.tmA0, a.a0_codes, true, a.K, rows_total, mr)) return cudaErrorInvalidValue;
  if (phase == 1 && !make_map(&prm.tmA1, a.a1_codes, true, a.K, rows_total, mr))
    return cudaErrorInvalidValue;
  if (!make_map(&prm.tmB, a.b_codes, false, a.K, a.R, 16)) return cudaErrorInvalidValue;
  prm.sfa0 = a.a0_scales;
  prm.sfa1 = a.a1_scales;
  prm.b_scales = a.b_scales;
  prm.plan = a.plan;
  prm.E = a.E;
  prm.K = a.K;
  prm.rows_per_expert = a.rows_per_expert;
  prm.R = a.R;
  prm.P = a.P;
  prm.f = a.f;
  prm.d = a.d;
  prm.qh = a.qh;
  prm.sh = a.sh;
  prm.y_routed = a.y_routed;
  prm.y_shared = a.y_shared;
  prm.wait_ns = a.wait_ns;
  prm.status = a.status;
  prm.counters = a.counters;
  prm.partials = a.partials;
  prm.ncap = a.ncap;
  prm.l2_hints = a.l2_hints;
  const int grid = num_sms < kMaxCtas ? num_sms : kMaxCtas;
#define X(P, N, S, B, M) \
  if (phase == P && nmax == N && mr == M) return launch_one<P, N, S, B, M>(prm, s, grid, a.overlap);
  BITMOE_FFN_VARIANTS(X)
#undef X
  return cudaErrorInvalidValue;
}

}  // namespace bitmoe
