// Batched decode path of the expert FFN (a few to 64 tokens): memory-bound FP4 GEMVs over
// groups of up to 8 tokens.
//
// With tens of tokens most active experts serve one or two of them, so the layer is still
// bound by reading every active expert's FP4 codes and block scales once (dpshk.com
// article, "核心实现三": an expert is read once for all its tokens; "核心实现四": FP4 is
// decoded inside the GEMV, gate and up share one quantised input).  The tcgen05 tile
// kernels cannot stream at that rate here: the block-scaled MMA reads FP4 only unpacked
// to a byte per element in shared memory, so a stage holds half the HBM bytes it would
// hold packed and too few bytes are in flight per SM.  These kernels keep the codes
// packed and decode them in registers (cvt e2m1x2 -> f16x2), with the tokens in the N = 8
// columns of mma.sync m16n8k16.
//
// Slots: the prepare kernel cuts every expert's token rows (routed pairs in expert-sorted
// order, then the shared expert's T rows) into slots of at most 8 rows (expert, first
// row, rows).  An expert with more than 8 tokens has several slots; each reads the
// expert's weights again, and those reads are marked evict-last so that the slots after
// the first find the weights in L2.
//
// Units (16 weight rows: phase 1 = 8 gate + the same 8 up rows, phase 2 = 16 down rows)
// of every slot, in slot order, are cut into one contiguous range per CTA.  A CTA's 16
// compute warps take its units round-robin, each unit whole: the warp streams the unit's
// 512-wide K stages through its private ring of 2 stages (TMA: 3-D code boxes with the
// 128-byte swizzle, 2-D scale boxes) and accumulates in registers, so the sum runs in K
// order: per 32-element block two MMAs (exact f16 products, fp32 sums), times the row's
// ue8m0 scale (exact), per 128-block times each token's fp32 activation scale.  A loader
// warp brings each slot's e4m3 activation rows (one 3-D TMA box, 128-byte swizzle) and
// their fp32 scales into one of two shared-memory buffers, reusing a buffer once every
// compute warp has passed its slot.
//
// Phase 1 writes h = silu(g) * u (fp32) per (token, h-row); a small kernel re-quantises h
// per 128-block (quant.cu); phase 2 reads those codes and writes fp32 y rows.  Every wait
// is bounded (%globaltimer); an expired wait records MOE_ERR_TIMEOUT, the warp lets its
// issued copies land, and the CTA returns.
#include "internal.cuh"
#include "ptx.cuh"
#include "waits.cuh"

#include <cstring>

namespace bitmoe {
namespace {

constexpr int kBgWarps = 16;                        // compute warps
constexpr int kBgThreads = (kBgWarps + 1) * 32;     // + the activation loader warp
constexpr int kBgStages = 2;                        // weight ring depth per warp
constexpr int kBgRows = 16;
constexpr int kBgCodeBytes = kBgRows * 256;
constexpr int kBgScaleBytes = kBgRows * 16;
constexpr int kBgStageBytes = kBgCodeBytes + kBgScaleBytes;
constexpr int kBgBufs = 2;                          // activation buffers
constexpr int kBgMaxCtaSlots = 64;                  // slots of one CTA's range
constexpr int kNT = kBgSlotTokens;                  // 8 tokens per slot

struct BgParams {
  CUtensorMap tm_c0, tm_s0, tm_c1, tm_s1;  // weights: gate, up (phase 1) or down (phase 2)
  CUtensorMap tm_act;                      // activation codes [R][K] (piece, row, piece index)
  CUtensorMap tm_asc;                      // activation scales [R][K/128] fp32
  const int32_t* plan;                     // [0] = slots, then (expert, first row, rows)
  float* hbuf;                             // phase 1 out: h [R][f] fp32
  float* y_routed;                         // phase 2 out: [P][d]
  float* y_shared;                         // phase 2 out: [T][d] (rows P..P+T-1)
  int E, K, rows_per_expert, P, R, d, f;
  long long wait_ns;
  int* status;
  FastDiv fd_s, fd_upe;  // stages per unit (K / 512), units per expert
};

// Shared memory from a 1024-byte aligned base.
struct BgSmem {
  int K;
  __host__ __device__ int act_bytes() const { return kNT * K; }  // one buffer of codes
  __host__ __device__ int off_asc() const { return kBgBufs * act_bytes(); }
  __host__ __device__ int off_ring() const {
    return (off_asc() + kBgBufs * kNT * (K / 128) * 4 + 1023) / 1024 * 1024;
  }
  __host__ __device__ int off_rscale() const { return off_ring() + kBgWarps * kBgStages * kBgCodeBytes; }
  __host__ __device__ int off_bars() const { return off_rscale() + kBgWarps * kBgStages * kBgScaleBytes; }
  // ring [warp][stage], act_full[buf], act_empty[buf]
  __host__ __device__ int off_info() const {
    return off_bars() + (kBgWarps * kBgStages + 2 * kBgBufs) * 8;
  }
  // abort, then (expert, first row, rows, evict-last) per slot of the range
  __host__ __device__ int bytes() const { return off_info() + 16 + kBgMaxCtaSlots * 16 + 1024; }
};

__device__ __forceinline__ void ue8m0x4_f32(uint32_t w, float (&f)[4]) {
  const uint32_t m = 0x7F800000u, e0 = 0x00400000u;
  f[0] = __uint_as_float(max((w << 23) & m, e0));
  f[1] = __uint_as_float(max((w << 15) & m, e0));
  f[2] = __uint_as_float(max((w << 7) & m, e0));
  f[3] = __uint_as_float(max((w >> 1) & m, e0));
}

// Stage layout of the weight codes: byte 4t of 32-block b (0..15) of stage row r (phase 1:
// rows 0-7 gate, 8-15 up, boxes [matrix][half][8 rows]; phase 2: boxes [half][16 rows]),
// 128-byte swizzle.
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

// Activation buffer layout [piece k/128][token row][128 bytes], 128-byte swizzle: bytes
// 8t..8t+7 of 32-block (k / 32) for token g.
__device__ __forceinline__ uint32_t act_offset(int k, int g, int t) {
  const int piece = k >> 7, chunk = ((k & 127) >> 4) + (t >> 1);
  return (uint32_t)piece * 1024u + (uint32_t)g * 128u + ((uint32_t)(chunk ^ g) << 4) +
         8u * (uint32_t)(t & 1);
}

// KC, RPE: 0 for the sizes of the launch, or K and the rows per expert fixed at compile time
// (the decode sizes' instantiations, whose work-split and layout arithmetic folds).
template <int PHASE, int KC = 0, int RPE = 0>
__global__ void __launch_bounds__(kBgThreads, 1) bgemv_kernel(const __grid_constant__ BgParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  const int K = KC ? KC : p.K;
  const int rpe = RPE ? RPE : p.rows_per_expert;
  const BgSmem L{K};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nb = K / 128;
  const uint32_t bars = ptx::smem_u32(smem + L.off_bars());
  auto full = [&](int s) { return bars + 8u * (uint32_t)(warp * kBgStages + s); };
  auto act_full = [&](int b) { return bars + 8u * (uint32_t)(kBgWarps * kBgStages + b); };
  auto act_empty = [&](int b) {
    return bars + 8u * (uint32_t)(kBgWarps * kBgStages + kBgBufs + b);
  };
  int* info = reinterpret_cast<int*>(smem + L.off_info());
  volatile int* abort_flag = info;
  int* slot_info = info + 4;  // [slot - first][4]
  const float* asc = reinterpret_cast<const float*>(smem + L.off_asc());

  if (threadIdx.x == 0) {
    ptx::prefetch_tmap(&p.tm_c0);
    ptx::prefetch_tmap(&p.tm_s0);
    if (PHASE == 1) {
      ptx::prefetch_tmap(&p.tm_c1);
      ptx::prefetch_tmap(&p.tm_s1);
    }
    ptx::prefetch_tmap(&p.tm_act);
    ptx::prefetch_tmap(&p.tm_asc);
    for (int b = 0; b < kBgBufs; ++b) {
      ptx::mbar_init(act_full(b), 1);
      ptx::mbar_init(act_empty(b), kBgWarps);
    }
    *abort_flag = 0;
  }
  if (lane == 0 && warp < kBgWarps)
    for (int s = 0; s < kBgStages; ++s) ptx::mbar_init(full(s), 1);
  ptx::fence_mbar_init();
  // the plan and the activation rows come from the kernels before this one
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  const int n_slots = __ldg(p.plan);
  const int rows_unit = PHASE == 1 ? 8 : 16;
  const int upe = rpe / rows_unit;
  const FastDiv fd_s = KC ? FastDiv(KC / 512) : p.fd_s;
  const FastDiv fd_upe = RPE ? FastDiv(RPE / (PHASE == 1 ? 8 : 16)) : p.fd_upe;
  const long long U = (long long)n_slots * upe;
  const int u_lo = (int)(blockIdx.x * U / gridDim.x);
  const int u_hi = (int)((blockIdx.x + 1) * U / gridDim.x);
  const int first = u_lo / upe;
  const int last = u_hi > u_lo ? (u_hi - 1) / upe : first - 1;
  const int n_my = last - first + 1;
  if (n_slots < 0 || n_slots > p.R || n_my > kBgMaxCtaSlots) {  // never produced by the plan
    if (threadIdx.x == 0) atomicOr(p.status, kStatusBadIndex);
    return;
  }
  for (int i = threadIdx.x; i < n_my; i += kBgThreads) {
    const int s = first + i;
    int e = __ldg(p.plan + 1 + 3 * s), row0 = __ldg(p.plan + 2 + 3 * s), n = __ldg(p.plan + 3 + 3 * s);
    if (e < 0 || e > p.E || row0 < 0 || n < 1 || n > kNT || row0 + n > p.R) {
      atomicOr(p.status, kStatusBadIndex);
      e = 0;
      row0 = 0;
      n = 0;  // nothing is stored for this slot
    }
    // several slots of one expert: keep its weights in L2 for the others
    const bool multi = (s > 0 && __ldg(p.plan + 1 + 3 * (s - 1)) == e) ||
                       (s + 1 < n_slots && __ldg(p.plan + 1 + 3 * (s + 1)) == e);
    slot_info[4 * i] = e;
    slot_info[4 * i + 1] = row0;
    slot_info[4 * i + 2] = n;
    slot_info[4 * i + 3] = multi ? 1 : 0;
  }
  __syncthreads();

  if (warp == kBgWarps) {
    // ------------------------------------------------ activation loader (lane 0)
    if (lane == 0) {
      const uint32_t tx = (uint32_t)(L.act_bytes() + kNT * nb * 4);
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < n_my && ok; ++i) {
        const int b = i % kBgBufs;
        if (i >= kBgBufs) {  // every compute warp has passed the slot this buffer held
          ok = wait_one(act_empty(b), (uint32_t)(i / kBgBufs - 1) & 1u, p.wait_ns, abort_flag,
                        p.status);
          if (!ok) break;
        }
        ptx::mbar_arrive_expect_tx(act_full(b), tx);
        const uint32_t dst = ptx::smem_u32(smem + b * L.act_bytes());
        const uint32_t dsc = ptx::smem_u32(smem + L.off_asc() + b * kNT * nb * 4);
        const int row0 = slot_info[4 * i + 1];
        ptx::tma_load_3d(dst, &p.tm_act, 0, row0, 0, act_full(b));
        ptx::tma_load_2d(dsc, &p.tm_asc, 0, row0, act_full(b));
        ++issued;
      }
      // every copy must land before the CTA can exit
      for (int i = issued - kBgBufs < 0 ? 0 : issued - kBgBufs; i < issued; ++i)
        drain_wait(act_full(i % kBgBufs), (uint32_t)(i / kBgBufs) & 1u);
    }
    __syncwarp();
    return;
  }

  // ------------------------------------------------ compute warps
  const int S = K / 512;
  const uint64_t pol_first = ptx::make_policy_evict_first();
  const uint64_t pol_last = ptx::make_policy_evict_last();
  const int n_units = u_hi - u_lo;
  const int my_units = n_units > warp ? (n_units - warp + kBgWarps - 1) / kBgWarps : 0;
  const int total = my_units * S;  // this warp's stages: (its q-th unit, chunk)
  auto codes_at = [&](int s) { return smem + L.off_ring() + (warp * kBgStages + s) * kBgCodeBytes; };
  auto scales_at = [&](int s) {
    return smem + L.off_rscale() + (warp * kBgStages + s) * kBgScaleBytes;
  };
  auto issue = [&](int i) {
    const int qi = fd_s.div(i);
    const int u = u_lo + warp + qi * kBgWarps, c = i - qi * S;
    const int ue = fd_upe.div(u);
    const int sl = ue - first;
    const int e = slot_info[4 * sl];
    const uint64_t pol = slot_info[4 * sl + 3] ? pol_last : pol_first;
    const int st = i % kBgStages;
    const uint32_t dc = ptx::smem_u32(codes_at(st)), ds = ptx::smem_u32(scales_at(st));
    ptx::mbar_arrive_expect_tx(full(st), kBgStageBytes);
    const int row = e * rpe + (u - ue * upe) * rows_unit;
    ptx::tma_load_3d_hint(dc, &p.tm_c0, 0, row, 2 * c, full(st), pol);
    ptx::tma_load_2d_hint(ds, &p.tm_s0, c * 16, row, full(st), pol);
    if (PHASE == 1) {
      ptx::tma_load_3d_hint(dc + 2048, &p.tm_c1, 0, row, 2 * c, full(st), pol);
      ptx::tma_load_2d_hint(ds + 128, &p.tm_s1, c * 16, row, full(st), pol);
    }
  };
  int issued = 0;
  if (lane == 0)
    for (; issued < kBgStages && issued < total; ++issued) issue(issued);
  issued = __shfl_sync(0xffffffffu, issued, 0);

  const int r0 = g, r1 = g + 8;
  int released = 0;  // slots of the range this warp has passed (act_empty arrivals)
  bool ok = true;
  int i = 0;
  for (int q = 0; q < my_units && ok; ++q) {
    const int u = u_lo + warp + q * kBgWarps;
    const int ue = fd_upe.div(u);
    const int sl = ue - first;
    const int uin = u - ue * upe;
    for (; released < sl; ++released)
      if (lane == 0) ptx::mbar_arrive(act_empty(released % kBgBufs));
    if (!wait_warp(act_full(sl % kBgBufs), (uint32_t)(sl / kBgBufs) & 1u, p.wait_ns, abort_flag,
                   p.status)) {
      ok = false;
      break;
    }
    const uint8_t* ab = smem + (sl % kBgBufs) * L.act_bytes();
    const float* sb = asc + (sl % kBgBufs) * kNT * nb;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};  // (row g, token 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1)
    for (int c = 0; c < S; ++c, ++i) {
      const int st = i % kBgStages;
      if (!wait_warp(full(st), (uint32_t)(i / kBgStages) & 1u, p.wait_ns, abort_flag, p.status)) {
        ok = false;
        break;
      }
      const uint8_t* cst = codes_at(st);
      const uint8_t* sst = scales_at(st);
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {  // 128-element block j = 4c + ii
        const int j = 4 * c + ii;
        float fa[4], fb[4];
        ue8m0x4_f32(*reinterpret_cast<const uint32_t*>(sst + r0 * 16 + 4 * ii), fa);
        ue8m0x4_f32(*reinterpret_cast<const uint32_t*>(sst + r1 * 16 + 4 * ii), fb);
        float pa0 = 0.f, pa1 = 0.f, pb0 = 0.f, pb1 = 0.f;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const int blk = 4 * ii + bb;
          const uint32_t wa = *reinterpret_cast<const uint32_t*>(cst + code_offset<PHASE>(r0, blk, t));
          const uint32_t wb = *reinterpret_cast<const uint32_t*>(cst + code_offset<PHASE>(r1, blk, t));
          uint32_t ha[4], hb[4];
          ptx::cvt_e2m1x8_f16(wa, ha);
          ptx::cvt_e2m1x8_f16(wb, hb);
          const uint2 xq = *reinterpret_cast<const uint2*>(ab + act_offset(128 * j + 32 * bb, g, t));
          const uint32_t x0 = ptx::cvt_e4m3x2_f16x2((uint16_t)(xq.x & 0xffffu));
          const uint32_t x1 = ptx::cvt_e4m3x2_f16x2((uint16_t)(xq.x >> 16));
          const uint32_t x2 = ptx::cvt_e4m3x2_f16x2((uint16_t)(xq.y & 0xffffu));
          const uint32_t x3 = ptx::cvt_e4m3x2_f16x2((uint16_t)(xq.y >> 16));
          float cb[4];
          ptx::mma_m16n8k16_f16_zero(cb, ha[0], hb[0], ha[1], hb[1], x0, x1);
          ptx::mma_m16n8k16_f16(cb, ha[2], hb[2], ha[3], hb[3], x2, x3);
          pa0 = fmaf(fa[bb], cb[0], pa0);
          pa1 = fmaf(fa[bb], cb[1], pa1);
          pb0 = fmaf(fb[bb], cb[2], pb0);
          pb1 = fmaf(fb[bb], cb[3], pb1);
        }
        const float s0 = sb[(2 * t) * nb + j], s1 = sb[(2 * t + 1) * nb + j];
        acc[0] = fmaf(s0, pa0, acc[0]);
        acc[1] = fmaf(s1, pa1, acc[1]);
        acc[2] = fmaf(s0, pb0, acc[2]);
        acc[3] = fmaf(s1, pb1, acc[3]);
      }
      __syncwarp();  // every lane is done with the stage: its buffer may be refilled
      if (issued < total) {
        if (lane == 0) issue(issued);
        ++issued;
      }
    }
    if (!ok) break;
    const int n = slot_info[4 * sl + 2], row0 = slot_info[4 * sl + 1];
    if (PHASE == 1) {  // h = silu(g) * u for (h-row uin*8 + g, tokens 2t, 2t+1)
#pragma unroll
      for (int tk = 0; tk < 2; ++tk) {
        const int tok = 2 * t + tk;
        if (tok < n) {
          const float gg = acc[tk], uu = acc[2 + tk];
          p.hbuf[(size_t)(row0 + tok) * p.f + uin * 8 + g] = __fdividef(gg, 1.0f + expf(-gg)) * uu;
        }
      }
    } else {  // y rows uin*16 + g and + 8 of tokens 2t, 2t+1
#pragma unroll
      for (int tk = 0; tk < 2; ++tk) {
        const int tok = 2 * t + tk;
        if (tok < n) {
          const int row = row0 + tok;
          float* yr = row < p.P ? p.y_routed + (size_t)row * p.d : p.y_shared + (size_t)(row - p.P) * p.d;
          yr[uin * 16 + g] = acc[tk];
          yr[uin * 16 + g + 8] = acc[2 + tk];
        }
      }
    }
  }
  if (!ok && lane == 0)  // let the copies this warp issued land before the CTA exits
    for (int r = i; r < issued; ++r) drain_wait(full(r % kBgStages), (uint32_t)(r / kBgStages) & 1u);
  // release every remaining slot of the range, so the loader never waits on this warp
  for (; released < n_my; ++released)
    if (lane == 0) ptx::mbar_arrive(act_empty(released % kBgBufs));
  __syncwarp();
}

template <int PHASE, int KC = 0, int RPE = 0>
cudaError_t launch_one(const BgParams& prm, cudaStream_t s, int grid, bool overlap) {
  const size_t smem = (size_t)BgSmem{prm.K}.bytes();
  auto kern = bgemv_kernel<PHASE, KC, RPE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kBgThreads), smem, s, overlap, prm);
}

}  // namespace

size_t bgemv_smem_bytes(int K) { return (size_t)BgSmem{K}.bytes(); }

cudaError_t launch_bgemv(int phase, const BgLaunch& a, cudaStream_t s, int num_sms) {
  BgParams p;
  memset(&p, 0, sizeof(p));
  const int K = phase == 1 ? a.d : a.f;
  const int rpe = phase == 1 ? a.f : a.d;
  const long long rows = (long long)(a.E + 1) * rpe;
  const int box_rows = phase == 1 ? 8 : 16;
  if (!make_code_map(&p.tm_c0, a.a0_codes, K / 2, rows, box_rows) ||
      !make_byte_map(&p.tm_s0, a.a0_scales, K / 32, rows, 16, box_rows))
    return cudaErrorInvalidValue;
  if (phase == 1 && (!make_code_map(&p.tm_c1, a.a1_codes, K / 2, rows, box_rows) ||
                     !make_byte_map(&p.tm_s1, a.a1_scales, K / 32, rows, 16, box_rows)))
    return cudaErrorInvalidValue;
  if (!make_code_map(&p.tm_act, a.act, K, a.R, kNT, K / 128) ||
      !make_f32_map(&p.tm_asc, a.act_scales, K / 128, a.R, kNT))
    return cudaErrorInvalidValue;
  p.plan = a.plan;
  p.hbuf = a.hbuf;
  p.y_routed = a.y_routed;
  p.y_shared = a.y_shared;
  p.E = a.E;
  p.K = K;
  p.rows_per_expert = rpe;
  p.P = a.P;
  p.R = a.R;
  p.d = a.d;
  p.f = a.f;
  p.wait_ns = a.wait_ns;
  p.status = a.status;
  p.fd_s = FastDiv((uint32_t)(K / 512));
  p.fd_upe = FastDiv((uint32_t)(rpe / (phase == 1 ? 8 : 16)));
  const int grid = num_sms < kMaxCtas ? num_sms : kMaxCtas;
  if (a.d == 4096 && a.f == 2048)  // the decode sizes' instantiations
    return phase == 1 ? launch_one<1, 4096, 2048>(p, s, grid, a.overlap)
                      : launch_one<2, 2048, 4096>(p, s, grid, a.overlap);
  return phase == 1 ? launch_one<1>(p, s, grid, a.overlap) : launch_one<2>(p, s, grid, a.overlap);
}

}  // namespace bitmoe
