// Pieces shared by the single-token layer kernels (decode.cu, decode_tc.cu): the routing
// of one token by one warp, the top-k of its E router scores and its gate weights
// w_j = sigmoid(s_j) / sum of the k sigmoids (tcti.cn post, "补齐软件栈缺失": the router
// picks k routed experts per token; ties go to the lower expert id, as in the oracle), and
// the split of a phase's weight units over the CTAs.
#pragma once
#include <cstdint>

namespace bitmoe {
namespace {

// One CTA's share of a phase.  A shared unit weighs wsh (1; 2 in the Q2 form, where it
// has twice the stages of a routed unit), a routed unit 1: M = (n_routed + wsh) * upe in
// all, CTA b taking the weight range [b*M/G, (b+1)*M/G).  Its first ns units are the
// shared expert's [s_lo, s_lo+ns) (s_lo = b*upe/G, a share that does not depend on the
// routing), the rest the routed units [r_lo, r_lo+nr) of the list that runs over the
// active routed experts in slot order (r_lo = b*M/G - wsh*s_lo).
struct Range {
  int s_lo, ns, r_lo, nr, upe;
  __host__ __device__ Range(int upe_, int n_routed, int G, int b, int wsh) {
    upe = upe_;
    s_lo = (int)((long long)b * upe / G);
    ns = (int)((long long)(b + 1) * upe / G) - s_lo;
    const long long M = (long long)(n_routed + wsh) * upe;
    const long long t_lo = b * M / G, t_hi = (b + 1) * M / G;
    r_lo = (int)(t_lo - (long long)wsh * s_lo);
    nr = (int)(t_hi - t_lo) - wsh * ns;
  }
  __host__ __device__ int units() const { return ns + nr; }
};

// The lane's scores (experts lane + 32 i), -inf past E: loaded on their own so that a
// kernel can issue the loads first and route later.
template <int PL>
__device__ __forceinline__ void load_scores(const float* __restrict__ scores, int E, int lane,
                                            float (&v)[PL]) {
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(scores + e) : -INFINITY;
  }
}
// Each lane holds experts lane + 32 i (i < PL, so E <= 32 PL).  k rounds of a warp arg-max
// on (value desc, index asc), as a max of order-preserving integer keys and then a min of
// the indices holding it (two warp reductions a round).  Outputs, in shared memory: for
// slot = the expert's rank among the k selected ids (its sorted position), slot_e[slot] =
// the expert and, if non-NULL, slot_row[slot] = slot and slot_n[slot] = 1; for pair j (the
// j-th largest score), pair_w[j] and pair_pos[j] = its slot.  If idx is non-NULL the
// routing and dispatch results go to global memory too (idx, w, perm, pos).
template <int PL>
__device__ __forceinline__ void route_token_warp(const float (&v)[PL], int E, int k, int lane,
                                                 int* slot_e, int* slot_row, int* slot_n,
                                                 float* pair_w, int* pair_pos, int32_t* idx,
                                                 float* w, int32_t* perm, int32_t* pos) {
  // keys: a larger score has a larger key (sign-magnitude to offset order); NaN and
  // padding get 0, below every number, so they are taken only after all numbers
  uint32_t key[PL];
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const uint32_t u = __float_as_uint(v[i] == 0.f ? 0.f : v[i]);  // -0 ties +0
    key[i] = (v[i] != v[i] || lane + 32 * i >= E) ? 0u : ((u & 0x80000000u) ? ~u : (u | 0x80000000u));
  }
  unsigned taken = 0;
  float sel_v = 0.f;
  int sel_i = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0u, bidx = 0xFFFFFFFFu;
#pragma unroll
    for (int i = 0; i < PL; ++i) {
      if (!((taken >> i) & 1u) && (key[i] > bk || bidx == 0xFFFFFFFFu)) {
        bk = key[i];
        bidx = (uint32_t)(lane + 32 * i);
      }
    }
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t imin = __reduce_min_sync(0xffffffffu, bk == kmax ? bidx : 0xFFFFFFFFu);
    if ((int)(imin & 31u) == lane) taken |= 1u << (imin >> 5);
    if (lane == j) {
      sel_v = __uint_as_float((kmax & 0x80000000u) ? (kmax ^ 0x80000000u) : ~kmax);
      sel_i = (int)imin;
    }
  }
  const float sig = lane < k ? 1.0f / (1.0f + expf(-sel_v)) : 0.0f;
  float sum = sig;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  // slot (= sorted position) of pair j: the number of selected experts below it
  int rank = 0;
  for (int j = 0; j < k; ++j) {
    const int ej = __shfl_sync(0xffffffffu, sel_i, j);
    rank += (lane < k && ej < sel_i) ? 1 : 0;
  }
  if (lane < k) {
    slot_e[rank] = sel_i;
    if (slot_row) slot_row[rank] = rank;
    if (slot_n) slot_n[rank] = 1;
    pair_w[lane] = sig / sum;
    pair_pos[lane] = rank;
    if (idx) {
      idx[lane] = sel_i;
      w[lane] = sig / sum;
      perm[rank] = lane;
      pos[lane] = rank;
    }
  }
}

// The same, loading the scores itself.
template <int PL>
__device__ __forceinline__ void route_token_warp(const float* __restrict__ scores, int E, int k,
                                                 int lane, int* slot_e, int* slot_row,
                                                 int* slot_n, float* pair_w, int* pair_pos,
                                                 int32_t* idx, float* w, int32_t* perm,
                                                 int32_t* pos) {
  float v[PL];
  load_scores<PL>(scores, E, lane, v);
  route_token_warp<PL>(v, E, k, lane, slot_e, slot_row, slot_n, pair_w, pair_pos, idx, w, perm, pos);
}

}  // namespace
}  // namespace bitmoe
