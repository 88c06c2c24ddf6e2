// Single-token decode path of the expert FFN: memory-bound FP4 GEMVs.
//
// At T = 1 every expert group holds the one token, so gate/up (phase 1) and down
// (phase 2) are matrix-vector products whose cost is reading each selected expert's FP4
// codes and block scales once (dpshk.com article, "核心实现三" and "核心实现四": an
// expert is read once for all its tokens, and FP4 is decoded inside the product, never
// expanded to a float matrix in memory).  The tcgen05 tile path would spend a
// 32-column MMA tile and a TMEM round trip per 128-K chunk on one useful column.
//
// Each warp streams 16 weight rows (phase 1: 8 gate rows and the same 8 up rows;
// phase 2: 16 down rows) through its own ring of shared-memory stages, filled by TMA:
// per matrix one 3-D box of codes (2 halves x rows x 128 bytes, 128-byte swizzle, so
// that the lanes' 4-byte reads of eight rows hit distinct banks) and one 2-D box of
// 16 scale bytes x rows.  A stage holds 512 K-elements, i.e. 16 blocks of 32 per row.
//
// Per 32-element block b the warp runs two mma.sync m16n8k16 (f16 in, fp32 accumulate)
// into a fresh accumulator: lane (g, t) decodes bytes 4t..4t+3 of the block in rows g
// and g+8 (cvt e2m1x2 -> f16x2, eight elements per row) and holds the activation's
// elements 8t..8t+7 of the block in the B fragment.  The MMA's K order is thus a
// permutation of the block, the same on both sides.  The fp32 block partial is then
// multiplied by 2^(e-127) (the row's ue8m0 scale; exact in fp32) times the activation's
// fp32 scale of its 128-block and added to the row's accumulator.
//
// Phase 1 ends with h = silu(g) * u per row (fp32, to a workspace buffer).  Phase 2
// quantises the h of its experts in its prologue (amax / 448, IEEE divide, e4m3 round
// to nearest even: the same rule as the activations) and writes fp32 y rows.
//
// Work split: the units (16-row blocks of every selected expert, in plan order) are cut
// into one contiguous range per CTA (148 CTAs, one per SM).  A range spans at most two
// experts, whose activations the CTA keeps in shared memory as f16 values.  The
// range's stages (unit, K-chunk) go round-robin to the CTA's 24 warps, so that every
// warp streams and no warp holds more than one stage beyond the others; each stage
// leaves its 16 row partials in shared memory, and after a CTA barrier the partials of
// each row are summed in K order (the result does not depend on timing).
#include "internal.cuh"
#include "ptx.cuh"
#include "waits.cuh"

#include <cstring>

namespace bitmoe {
namespace {

constexpr int kGvWarps = 24;
constexpr int kGvThreads = kGvWarps * 32;
constexpr int kGvStages = 2;                          // ring depth per warp
constexpr int kGvRows = 16;                           // weight rows per unit
constexpr int kGvCodeBytes = kGvRows * 256;           // 256 code bytes (512 elements) per row
constexpr int kGvScaleBytes = kGvRows * 16;           // 16 ue8m0 bytes per row
constexpr int kGvStageBytes = kGvCodeBytes + kGvScaleBytes;
constexpr int kGvMaxSlots = 2;                        // experts per CTA range
constexpr int kGvMaxUnits = 16;                       // units per CTA range
constexpr int kGvPlanInts = 3 + 2 * (kMaxCtas - 1);   // plan words read (<= kMaxCtas experts)

struct GemvParams {
  CUtensorMap tm_c0;         // gate (phase 1) or down (phase 2) codes [rows][K/2], experts stacked
  CUtensorMap tm_s0;         // their scales [rows][K/32]
  CUtensorMap tm_c1;         // up codes and scales (phase 1)
  CUtensorMap tm_s1;
  const int32_t* plan;       // [0] = active experts n, then n pairs (expert, output row)
  const uint8_t* qx;         // phase 1: the token's e4m3 codes [K]
  const float* sx;           // phase 1: its block scales [K/128]
  float* hbuf;               // phase 1 out, phase 2 in: h [slot][f] fp32
  float* y_routed;           // phase 2 out: y rows [T*k][d] (expert-sorted order)
  float* y_shared;           // phase 2 out: the shared expert's row [d]
  uint8_t* qh;               // phase 2 out: the re-quantised h [row][f] e4m3 and its
  float* sh;                 //   scales [row][f/128] (row = output row, P for the shared)
  int E, K, rows_per_expert, f, d, P;
  long long wait_ns;
  int* status;
  int stall;                 // test knob: warp 0 of CTA 0 waits on a barrier nothing completes
};

// Shared memory (from a 1024-byte aligned base): code rings [warp][stage] (each stage
// 4 KB, 1024-aligned for the swizzled boxes), scale rings, activations (phase 1: the
// token; phase 2: up to two experts' h), stage partials [unit][K-chunk][16 rows],
// barriers.
struct GvSmem {
  static constexpr int kOffScales = kGvWarps * kGvStages * kGvCodeBytes;
  static constexpr int kOffB = kOffScales + kGvWarps * kGvStages * kGvScaleBytes;
  // activation rows held: phase 1 has the one token for every expert
  __host__ __device__ static int slots(int phase) { return phase == 1 ? 1 : kGvMaxSlots; }
  __host__ __device__ static int off_bs(int phase, int K) { return kOffB + slots(phase) * K * 2; }
  __host__ __device__ static int off_part(int phase, int K) {
    return off_bs(phase, K) + slots(phase) * (K / 128) * 4;
  }
  __host__ __device__ static int off_bars(int phase, int K) {
    return off_part(phase, K) + kGvMaxUnits * (K / 512) * kGvRows * 4;
  }
  __host__ __device__ static int off_plan(int phase, int K) {
    return off_bars(phase, K) + kGvWarps * kGvStages * 8;
  }
  __host__ __device__ static int off_misc(int phase, int K) {
    return off_plan(phase, K) + kGvPlanInts * 4;
  }
  // misc: abort flag, then (expert, output row) of the range's slots, then (8-byte
  // aligned) the barrier the test stall waits on
  __host__ __device__ static int off_stall(int phase, int K) {
    return (off_misc(phase, K) + 32 + 7) / 8 * 8;
  }
  __host__ __device__ static size_t bytes(int phase, int K) {
    return (size_t)off_misc(phase, K) + 48 + 1024;
  }
};

// 2^(e-127) in fp32 for the four ue8m0 bytes of w (byte 0 first; 2^-127 is a subnormal)
__device__ __forceinline__ void ue8m0x4_f32(uint32_t w, float (&f)[4]) {
  const uint32_t m = 0x7F800000u, e0 = 0x00400000u;
  f[0] = __uint_as_float(max((w << 23) & m, e0));
  f[1] = __uint_as_float(max((w << 15) & m, e0));
  f[2] = __uint_as_float(max((w << 7) & m, e0));
  f[3] = __uint_as_float(max((w >> 1) & m, e0));
}

// Byte offset, in a stage, of bytes 4t..4t+3 of block b (0..15) of stage row r.  Row r
// lies in box (matrix, half b/8) at box row rb; the 128-byte swizzle XORs the 16-byte
// chunk index with the row index mod 8.
template <int PHASE>
__device__ __forceinline__ uint32_t code_offset(int r, int b, int t) {
  const int half = b >> 3, chunk = b & 7;
  uint32_t box, rb;
  if (PHASE == 1) {  // rows 0-7 gate, 8-15 up; boxes of 8 rows: [matrix][half]
    box = (uint32_t)((r >> 3) * 2 + half) * 1024u;
    rb = (uint32_t)(r & 7);
  } else {           // boxes of 16 rows: [half]
    box = (uint32_t)half * 2048u;
    rb = (uint32_t)r;
  }
  return box + rb * 128u + ((uint32_t)(chunk ^ (r & 7)) << 4) + 4u * (uint32_t)t;
}

template <int PHASE>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_kernel(const __grid_constant__ GemvParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  const int K = p.K;
  uint16_t* bx = reinterpret_cast<uint16_t*>(smem + GvSmem::kOffB);        // [slot][K] f16
  float* bs = reinterpret_cast<float*>(smem + GvSmem::off_bs(PHASE, K));    // [slot][K/128]
  float* part = reinterpret_cast<float*>(smem + GvSmem::off_part(PHASE, K));
  const uint32_t bars = ptx::smem_u32(smem + GvSmem::off_bars(PHASE, K));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + GvSmem::off_misc(PHASE, K));
  int* slot_info = reinterpret_cast<int*>(smem + GvSmem::off_misc(PHASE, K) + 16);  // [slot][2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  auto full = [&](int s) { return bars + 8u * (uint32_t)(warp * kGvStages + s); };
  auto codes_at = [&](int s) { return smem + (warp * kGvStages + s) * kGvCodeBytes; };
  auto scales_at = [&](int s) {
    return smem + GvSmem::kOffScales + (warp * kGvStages + s) * kGvScaleBytes;
  };

  if (threadIdx.x == 0) {  // kernel parameters: fetch the descriptors before the wait
    ptx::prefetch_tmap(&p.tm_c0);
    ptx::prefetch_tmap(&p.tm_s0);
    if (PHASE == 1) {
      ptx::prefetch_tmap(&p.tm_c1);
      ptx::prefetch_tmap(&p.tm_s1);
    }
  }
  if (lane == 0)
    for (int s = 0; s < kGvStages; ++s) ptx::mbar_init(full(s), 1);
  const uint32_t stall_bar = ptx::smem_u32(smem + GvSmem::off_stall(PHASE, K));
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    ptx::mbar_init(stall_bar, 1);  // never arrived on: only the test stall waits on it
  }
  ptx::fence_mbar_init();

  // The plan comes from the prepare kernel, the activations of phase 1 too, and phase 2's
  // h from the gate/up kernel.  Phase 2 runs after gate/up, which passes its own wait
  // (so the prepare kernel has completed) before it lets this grid start: phase 2 reads
  // the plan and starts its weight copies first, and waits only before reading h.
  if (PHASE == 1) {
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
  }

  // one round trip to L2: the plan words (count + at most P + 1 pairs) and, in phase 1,
  // the token's codes (16 per thread) and block scales
  int* plan_s = reinterpret_cast<int*>(smem + GvSmem::off_plan(PHASE, K));
  const int plan_len = min(3 + 2 * p.P, kGvPlanInts);
  const int nb = K / 128;
  for (int i = threadIdx.x; i < plan_len; i += kGvThreads) plan_s[i] = p.plan[i];
  uint4 qv = make_uint4(0, 0, 0, 0);
  float sxv = 0.f;
  if (PHASE == 1) {
    if ((int)threadIdx.x < K / 16) qv = *reinterpret_cast<const uint4*>(p.qx + 16 * threadIdx.x);
    if ((int)threadIdx.x < nb) sxv = p.sx[threadIdx.x];
  }
  __syncthreads();
  const int n_act = plan_s[0];
  const int rows_unit = PHASE == 1 ? kGvRows / 2 : kGvRows;
  const int upe = p.rows_per_expert / rows_unit;  // units per expert
  const int N = n_act * upe;
  const int u_lo = (int)((long long)blockIdx.x * N / gridDim.x);
  const int u_hi = (int)((long long)(blockIdx.x + 1) * N / gridDim.x);
  const int n_units = u_hi - u_lo;
  const int S = K / 512;                           // stages (K-chunks) per unit
  const int n_tasks = n_units * S;
  const int total = n_tasks > warp ? (n_tasks - warp + kGvWarps - 1) / kGvWarps : 0;
  const int slot_lo = u_lo / upe;
  const int n_slots = n_units > 0 ? (u_hi - 1) / upe - slot_lo + 1 : 0;
  // the host keeps every range within kGvMaxUnits units and kGvMaxSlots experts; a
  // plan that breaks it is flagged, and the CTA stops before any copy
  if (n_act < 0 || n_act > p.P + 1 || 1 + 2 * n_act > plan_len || n_units > kGvMaxUnits ||
      n_slots > kGvMaxSlots) {
    if (threadIdx.x == 0) atomicOr(p.status, kStatusBadIndex);
    return;
  }
  if (threadIdx.x < n_slots) {
    int e = plan_s[1 + 2 * (slot_lo + threadIdx.x)];
    int orow = plan_s[2 + 2 * (slot_lo + threadIdx.x)];
    if (e < 0 || e > p.E || orow >= p.P) {  // never produced by the prepare kernel
      atomicOr(p.status, kStatusBadIndex);
      e = 0;
      orow = -2;  // nothing is stored for this slot
    }
    slot_info[2 * threadIdx.x] = e;
    slot_info[2 * threadIdx.x + 1] = orow;
  }
  __syncthreads();

  const uint64_t pol = ptx::make_policy_evict_first();

  // the q-th stage of this warp is task warp + q * kGvWarps: unit u_lo + task / S,
  // K-chunk task % S; lane 0 issues its copies
  auto issue = [&](int q) {
    const int task = warp + q * kGvWarps;
    const int u = u_lo + task / S;
    const int c = task % S;
    const int e = slot_info[2 * (u / upe - slot_lo)];
    const int st = q % kGvStages;
    const uint32_t dc = ptx::smem_u32(codes_at(st)), ds = ptx::smem_u32(scales_at(st));
    ptx::mbar_arrive_expect_tx(full(st), kGvStageBytes);
    const int xs = c * 16;
    if (PHASE == 1) {
      const int row = e * p.rows_per_expert + (u % upe) * 8;
      ptx::tma_load_3d_hint(dc, &p.tm_c0, 0, row, 2 * c, full(st), pol);
      ptx::tma_load_3d_hint(dc + 2048, &p.tm_c1, 0, row, 2 * c, full(st), pol);
      ptx::tma_load_2d_hint(ds, &p.tm_s0, xs, row, full(st), pol);
      ptx::tma_load_2d_hint(ds + 128, &p.tm_s1, xs, row, full(st), pol);
    } else {
      const int row = e * p.rows_per_expert + (u % upe) * 16;
      ptx::tma_load_3d_hint(dc, &p.tm_c0, 0, row, 2 * c, full(st), pol);
      ptx::tma_load_2d_hint(ds, &p.tm_s0, xs, row, full(st), pol);
    }
  };

  int issued = 0;
  if (lane == 0)
    for (; issued < kGvStages && issued < total; ++issued) issue(issued);
  issued = __shfl_sync(0xffffffffu, issued, 0);

  if (PHASE == 2) {
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
  }

  // activations of this CTA's experts -> f16 values and fp32 block scales
  if (PHASE == 1) {
    for (int i = threadIdx.x; i < K / 16; i += kGvThreads) {
      const uint4 v = i == (int)threadIdx.x ? qv : *reinterpret_cast<const uint4*>(p.qx + 16 * i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[8];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        o[2 * h] = ptx::cvt_e4m3x2_f16x2((uint16_t)(w[h] & 0xffffu));
        o[2 * h + 1] = ptx::cvt_e4m3x2_f16x2((uint16_t)(w[h] >> 16));
      }
      uint4* dst = reinterpret_cast<uint4*>(bx + 16 * i);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    for (int i = threadIdx.x; i < nb; i += kGvThreads)
      bs[i] = i == (int)threadIdx.x ? sxv : p.sx[i];
  } else {
    // one warp per 128-block: 4 consecutive h values per lane
    for (int w = warp; w < n_slots * nb; w += kGvWarps) {
      const int sl = w / nb, j = w % nb;
      const float4 h = *reinterpret_cast<const float4*>(p.hbuf + (size_t)(slot_lo + sl) * K +
                                                        128 * j + 4 * lane);
      float amax = fmaxf(fmaxf(fabsf(h.x), fabsf(h.y)), fmaxf(fabsf(h.z), fabsf(h.w)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float sc = amax == 0.f ? 1.0f : __fdiv_rn(amax, 448.0f);
      const uint16_t q01 = ptx::cvt_e4m3x2(__fdiv_rn(h.x, sc), __fdiv_rn(h.y, sc));
      const uint16_t q23 = ptx::cvt_e4m3x2(__fdiv_rn(h.z, sc), __fdiv_rn(h.w, sc));
      uint32_t* dst = reinterpret_cast<uint32_t*>(bx + (size_t)sl * K + 128 * j + 4 * lane);
      dst[0] = ptx::cvt_e4m3x2_f16x2(q01);
      dst[1] = ptx::cvt_e4m3x2_f16x2(q23);
      if (lane == 0) bs[sl * nb + j] = sc;
      // the CTA whose range starts the expert's units also stores the codes and scales
      if ((slot_lo + sl) * upe >= u_lo && slot_info[2 * sl + 1] >= -1) {
        const int orow = slot_info[2 * sl + 1];
        const size_t row = orow >= 0 ? (size_t)orow : (size_t)p.P;
        *reinterpret_cast<uint32_t*>(p.qh + row * K + 128 * j + 4 * lane) =
            (uint32_t)q01 | ((uint32_t)q23 << 16);
        if (lane == 0) p.sh[row * nb + j] = sc;
      }
    }
  }
  __syncthreads();

  const int r0 = g, r1 = g + 8;  // this lane's stage rows (phase 1: gate g, up g)
  bool ok = true;
  int q = 0;
  for (; q < total; ++q) {
    const int st = q % kGvStages;
    // test stall: a wait that no copy completes, so that its time limit runs out
    if (p.stall && blockIdx.x == 0 && warp == 0 && q == 0 &&
        !wait_warp(stall_bar, 0, p.wait_ns, abort_flag, p.status)) {
      ok = false;
      break;
    }
    if (!wait_warp(full(st), (uint32_t)(q / kGvStages) & 1u, p.wait_ns, abort_flag, p.status)) {
      ok = false;
      break;
    }
    const int task = warp + q * kGvWarps;
    const int ul = task / S, c = task % S;
    const int sl = (u_lo + ul) / upe - slot_lo;
    const uint8_t* cst = codes_at(st);
    const uint8_t* sst = scales_at(st);
    const uint16_t* xb = bx + (PHASE == 1 ? 0 : (size_t)sl * K);
    const float* sxb = bs + (PHASE == 1 ? 0 : sl * nb);
    float acc0 = 0.f, acc1 = 0.f;  // rows g and g+8, column 0
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // 128-element activation block j = 4c + i
      const int j = 4 * c + i;
      float fa[4], fb[4];
      ue8m0x4_f32(*reinterpret_cast<const uint32_t*>(sst + r0 * 16 + 4 * i), fa);
      ue8m0x4_f32(*reinterpret_cast<const uint32_t*>(sst + r1 * 16 + 4 * i), fb);
      float pa = 0.f, pb = 0.f;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const int b = 4 * i + bb;  // block within the stage
        const uint32_t wa = *reinterpret_cast<const uint32_t*>(cst + code_offset<PHASE>(r0, b, t));
        const uint32_t wb = *reinterpret_cast<const uint32_t*>(cst + code_offset<PHASE>(r1, b, t));
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
    // every value read from the stage has been consumed above, so once all lanes are
    // past this point the next TMA copy may overwrite it
    __syncwarp();
    if (issued < total) {
      if (lane == 0) issue(issued);
      ++issued;
    }
    // column 0 (the token) sits in lanes t == 0
    if (t == 0) {
      float* pp = part + (ul * S + c) * kGvRows;
      pp[r0] = acc0;
      pp[r1] = acc1;
    }
  }
  if (!ok) {  // let the copies still in flight land before the CTA exits
    if (lane == 0)
      for (int r = q; r < issued; ++r)
        drain_wait(full(r % kGvStages), (uint32_t)(r / kGvStages) & 1u);
    __syncwarp();
  }
  __syncthreads();

  // each row: its stage partials summed in K order
  if (PHASE == 1) {
    for (int idx = threadIdx.x; idx < n_units * 8; idx += kGvThreads) {
      const int ul = idx >> 3, r = idx & 7;
      float gg = 0.f, uu = 0.f;
      for (int c = 0; c < S; ++c) {
        gg += part[(ul * S + c) * kGvRows + r];
        uu += part[(ul * S + c) * kGvRows + 8 + r];
      }
      const int u = u_lo + ul;
      const float h = __fdividef(gg, 1.0f + expf(-gg)) * uu;
      p.hbuf[(size_t)(u / upe) * p.f + (size_t)(u % upe) * 8 + r] = h;
    }
  } else {
    for (int idx = threadIdx.x; idx < n_units * kGvRows; idx += kGvThreads) {
      const int ul = idx >> 4, r = idx & 15;
      float y = 0.f;
      for (int c = 0; c < S; ++c) y += part[(ul * S + c) * kGvRows + r];
      const int u = u_lo + ul;
      const int orow = slot_info[2 * (u / upe - slot_lo) + 1];
      if (orow >= -1) {
        float* yr = orow >= 0 ? p.y_routed + (size_t)orow * p.d : p.y_shared;
        yr[(size_t)(u % upe) * 16 + r] = y;
      }
    }
  }
}


}  // namespace

size_t gemv_smem_bytes(int phase, int K) { return GvSmem::bytes(phase, K); }

int gemv_max_units_per_cta() { return kGvMaxUnits; }

cudaError_t launch_gemv(int phase, const GemvLaunch& a, cudaStream_t s, int num_sms) {
  GemvParams p;
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
  p.plan = a.plan;
  p.qx = a.qx;
  p.sx = a.sx;
  p.hbuf = a.hbuf;
  p.y_routed = a.y_routed;
  p.y_shared = a.y_shared;
  p.qh = a.qh;
  p.sh = a.sh;
  p.E = a.E;
  p.K = K;
  p.rows_per_expert = rpe;
  p.f = a.f;
  p.d = a.d;
  p.P = a.P;
  p.wait_ns = a.wait_ns;
  p.status = a.status;
  p.stall = a.stall;
  const size_t smem = GvSmem::bytes(phase, p.K);
  auto kern = phase == 1 ? gemv_kernel<1> : gemv_kernel<2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = num_sms < kMaxCtas ? num_sms : kMaxCtas;
  return launch_pdl(kern, dim3(grid), dim3(kGvThreads), smem, s, a.overlap, p);
}

}  // namespace bitmoe
