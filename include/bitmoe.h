/*
 * bitmoe — routed-expert FFN of one DeepSeek-V4-Flash-style MoE layer on B200 (sm_100a).
 *
 * C ABI of libbitmoe.so.  The pages this library follows:
 *  [P1] "DeepSeek-V4-Flash on 4x RTX 2080 Ti" forum post (tcti.cn):
 *       section "DeepSeek-V4-Flash的可能性" — routed experts stored as FP4, top-6 of
 *       256 routed experts per token, an always-on shared expert;
 *       section "补齐软件栈缺失" — act_quant (activation quantisation for the FP8/FP4
 *       linears) and fp4_gemm (FP8-quantised activation x FP4 packed weight);
 *       prefill is compute-bound and decode memory-bound, so they need different
 *       operators.
 *  [P2] "deepseek-v4-flash-0731-in-c" article (dpshk.com):
 *       section "核心实现一：MoE 专家流式读取" — the router picks each token's experts;
 *       section "核心实现三：多 token 批处理" — an expert's weights are read once for
 *       every token routed to it;
 *       section "核心实现四：低比特融合算子" — FP4 is dequantised inside the GEMV, never
 *       expanded to a float matrix; gate and up share one quantised input;
 *       workspaces are preallocated and reused.
 *
 * Numeric contract (what the pages leave open, fixed here):
 *   T tokens, E routed experts + 1 shared expert (index E), top-k routing,
 *   hidden size d, expert width f (d, f multiples of 128).
 *   Weights per expert: W_gate, W_up [f][d] and W_down [d][f], FP4 e2m1 codes packed
 *   two per byte (low nibble = even element), one ue8m0 scale byte (2^(b-127)) per 32
 *   consecutive elements along the reduction axis: codes [rows][K/2], scales [rows][K/32].
 *   Activations: per token and 128-element block, s = amax/448 (fp32, 1 if amax = 0),
 *   q = e4m3(x/s) rounded to nearest even, saturating at +-448.
 *   g = W_gate x^, u = W_up x^, h = silu(g) * u (fp32), h re-quantised like x,
 *   y = W_down h^.  Combine: out[t] = y_shared[t] + sum_j w[t,j] y[t,j] with
 *   w[t,j] = sigmoid(s_j) / sum_j' sigmoid(s_j') over the k selected scores.
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE pointers owned by the caller; the library never
 *     allocates or frees memory on these calls and never synchronises the stream.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); work is enqueued on it.
 *   - Return 0 (MOE_OK) or a negative MOE_ERR_* code; moe_last_error() gives a
 *     thread-local message for the last failing call on the calling thread.
 *   - T == 0 is a valid no-op.
 *   - Errors found on the device (a bounded wait that expired) are recorded in a
 *     device-side status word and returned by moe_sync_status().
 *   - On first use on a device the library looks up and keeps the device addresses of its
 *     own device variables (the status word, the single-token kernel's grid barrier, the
 *     scratch of moe_expert_ffn_noalloc).  cudaDeviceReset unloads them: after a reset,
 *     make no further call of this library on that device in the same process.
 */
#ifndef BITMOE_H
#define BITMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1) /* null / misaligned pointer, bad size or shape */
#define MOE_ERR_WORKSPACE (-2)   /* workspace smaller than moe_workspace_size() */
#define MOE_ERR_CUDA (-3)        /* a CUDA launch or driver call failed */
#define MOE_ERR_TIMEOUT (-4)     /* a bounded device-side wait expired */
#define MOE_ERR_UNSUPPORTED (-5) /* the current device is not sm_100 */

/* One layer's weights, E+1 experts (index E = shared expert), contiguous per matrix:
 *   gate_codes, up_codes  [E+1][f][d/2]   gate_scales, up_scales  [E+1][f][d/32]
 *   down_codes            [E+1][d][f/2]   down_scales             [E+1][d][f/32]
 * Code arrays must be 32-byte aligned; scale arrays 4-byte aligned. */
typedef struct {
  const uint8_t* gate_codes;
  const uint8_t* gate_scales;
  const uint8_t* up_codes;
  const uint8_t* up_scales;
  const uint8_t* down_codes;
  const uint8_t* down_scales;
  int E;
  int d;
  int f;
} moe_weights_t;

/* Step 1 — routing ([P1] "DeepSeek-V4-Flash的可能性": top-6 of 256 per token;
 * [P2] "核心实现一": the router decides each token's experts).
 *   scores   [T][E] fp32, finite.
 *   topk_idx [T][k] int32 out: the k largest scores, descending; equal scores go to
 *            the lower expert index.
 *   topk_w   [T][k] fp32 out: sigmoid(score) renormalised over the k selected.
 * 1 <= k <= min(E, 32); 1 <= E <= 1024.  Scores must be 4-byte aligned. */
int moe_route_topk(const float* scores, int T, int E, int k, int32_t* topk_idx,
                   float* topk_w, void* stream);

/* Router scoring + step 1 ([P2] "核心实现一": the router decides each token's experts
 * from its hidden state): scores[t][e] = x[t] . W_router[e], summed in fp32 over bf16
 * inputs, then the top-k of moe_route_topk on those scores.
 *   x_bf16        [T][d] bf16 bit patterns; w_router_bf16 [E][d] bf16.
 *   scores        [T][E] fp32 out (the router scores the selection used).
 *   topk_idx, topk_w as for moe_route_topk.
 * d % 128 == 0; 1 <= k <= min(E, 32); 1 <= E <= 1024; pointers 4-byte aligned.
 * Two kernels: the scores (tiles of 16 tokens x 8 experts, bf16 mma.sync, fp32 sums in a
 * fixed order), then top-k. */
int moe_router_topk(const uint16_t* x_bf16, const uint16_t* w_router_bf16, int T, int d, int E,
                    int k, float* scores, int32_t* topk_idx, float* topk_w, void* stream);

/* Step 2 — dispatch ([P2] "核心实现三": group tokens by expert so each expert's
 * weights are read once for its whole group).  Stable counting sort of the T*k
 * (token, slot) pairs, flat id p = t*k + j, by expert.
 *   counts  [E]   int32 out: pairs per expert.
 *   offsets [E+1] int32 out: exclusive prefix sum of counts (offsets[E] = T*k).
 *   perm    [T*k] int32 out: perm[r] = flat id at sorted position r; pairs of one
 *           expert keep ascending flat-id order.
 *   pos     [T*k] int32 out: inverse of perm.
 * topk_idx values must lie in [0, E).
 * ws/ws_bytes: optional scratch (may be NULL/0).  With at least
 * moe_dispatch_workspace_size(T, k, E) bytes (nonzero from 8192 pairs up), a large batch
 * runs a multi-CTA form (per-segment counts, then a scatter) instead of one CTA; the
 * result is the same permutation.  The scratch needs no initial contents. */
int moe_dispatch(const int32_t* topk_idx, int T, int k, int E, int32_t* counts,
                 int32_t* offsets, int32_t* perm, int32_t* pos, void* ws, size_t ws_bytes,
                 void* stream);

/* Step 3 — activation quantisation ([P1] "补齐软件栈缺失": act_quant).
 *   x_bf16 [T][d] bf16 bit patterns (16-byte aligned rows); qx [T][d] e4m3 codes out;
 *   sx [T][d/128] fp32 out.  d % 128 == 0, d <= 16384. */
int moe_act_quant(const uint16_t* x_bf16, int T, int d, uint8_t* qx, float* sx,
                  void* stream);

/* Steps 3-7 — expert FFN for every routed pair and the shared expert
 * ([P1] "补齐软件栈缺失": fp4_gemm; [P2] "核心实现四": fused FP4 dequantisation,
 * gate and up on one quantised input).  Quantises x, then for each expert runs
 * gate+up (block-scaled FP4 x FP8 tcgen05 MMA), SwiGLU and e4m3 re-quantisation of h,
 * then the down projection, reading each active expert's weights once per token tile.
 *   x_bf16   [T][d] bf16.   offsets [E+1], perm [T*k] from moe_dispatch.
 *   y_routed [T*k][d] fp32 out, row r = pair perm[r] (expert-sorted order).
 *   y_shared [T][d] fp32 out, the shared expert's output per token.
 *   ws       workspace of at least moe_workspace_size(T, k, E, d, f) bytes, 256-byte
 *            aligned; its contents need not be initialised.
 * k >= 1; d, f multiples of 128; d/2 and f/2 multiples of 32 (TMA row pitch). */
int moe_expert_ffn(const uint16_t* x_bf16, int T, int k, const moe_weights_t* w,
                   const int32_t* offsets, const int32_t* perm, float* y_routed,
                   float* y_shared, void* ws, size_t ws_bytes, void* stream);

/* The three stages moe_expert_ffn enqueues, exposed so that each can be timed alone.
 * Calling them in order with the same arguments is identical to moe_expert_ffn. */
int moe_ffn_prepare(const uint16_t* x_bf16, int T, int k, const moe_weights_t* w,
                    const int32_t* offsets, const int32_t* perm, void* ws, size_t ws_bytes,
                    void* stream);
int moe_ffn_gate_up(int T, int k, const moe_weights_t* w, void* ws, size_t ws_bytes,
                    void* stream);
int moe_ffn_down(int T, int k, const moe_weights_t* w, float* y_routed, float* y_shared,
                 void* ws, size_t ws_bytes, void* stream);

/* moe_expert_ffn without a caller-owned workspace.  The pages have no counterpart of
 * this call; it exists for callers that cannot allocate device memory when they run the
 * layer (an engine plugin given no workspace, a serving loop that must not call
 * cudaMalloc because it may synchronise the device).  Arguments and results are those of
 * moe_expert_ffn minus ws/ws_bytes; the scratch is a fixed array of
 * MOE_NOALLOC_SCRATCH_BYTES that the library keeps on every GPU that loads it, for the
 * life of the process.
 *   - Calls needing more scratch than that (moe_workspace_size > the maximum; for
 *     d = 4096, f = 2048, k = 6, E = 256 that is T > 72) return MOE_ERR_WORKSPACE.
 *   - Allocates nothing.  All calls share the one array per device: calls that overlap on
 *     the GPU (other streams, other threads) race on it.  It keeps the previous call's
 *     contents; nothing in it needs to start at zero.
 *   - The first call on a device looks up the array's device address once
 *     (cudaGetSymbolAddress) and fails with MOE_ERR_CUDA if that lookup fails. */
#define MOE_NOALLOC_SCRATCH_BYTES (24u << 20)
int moe_expert_ffn_noalloc(const uint16_t* x_bf16, int T, int k, const moe_weights_t* w,
                           const int32_t* offsets, const int32_t* perm, float* y_routed,
                           float* y_shared, void* stream);

/* Steps 1-8 in one call: route, dispatch, expert FFN and combine for T tokens, with the
 * arguments, outputs and rules of the four calls above (the outputs are the same arrays:
 * topk_idx [T][k], topk_w [T][k], counts [E], offsets [E+1], perm [T*k], pos [T*k],
 * y_routed [T*k][d], y_shared [T][d], out [T][d]; ws as for moe_expert_ffn).  The pages
 * describe the layer as this one sequence ([P2] "核心实现一" to "核心实现四").
 * A single token (T = 1; d, f multiples of 512; scale arrays 16-byte aligned; k <= 32)
 * runs as ONE cooperative kernel: routing, dispatch, quantisation, both FP4 GEMVs and
 * the combine, streaming the selected experts' weights from its first instruction.  Its
 * results equal those of the four calls bit for bit.  It needs every SM of the device for
 * the duration of the kernel (one block per SM, all resident at once), which a launch
 * under MPS limits or beside other resident work may not get: such a launch fails with
 * MOE_ERR_CUDA (cooperative launch too large) instead of running.  Larger batches run the
 * four calls back to back, each kernel after the first allowed to start under the tail
 * of the one before it.  k <= 32. */
int moe_forward(const float* scores, const uint16_t* x_bf16, int T, int k,
                const moe_weights_t* w, int32_t* topk_idx, float* topk_w, int32_t* counts,
                int32_t* offsets, int32_t* perm, int32_t* pos, float* y_routed, float* y_shared,
                float* out, void* ws, size_t ws_bytes, void* stream);

/* 2-bit routed experts (NEXT-2): the ai-muninn.com post "一張 22G 老卡跑 284B" runs the
 * model with its routed experts at 2 bits per weight (IQ2_XXS, 2.0625 bpw) and the
 * always-resident weights, the shared expert among them, at higher precision (the
 * smzdm.com post's "2-bit routed experts only" of the ds4 engine is the same split).  The
 * pages fix the bit rate, not the code book; this library's 2-bit codec is: four 2-bit
 * codes per byte (element i of a byte in bits 2i..2i+1), value code - 1.5 (-1.5, -0.5,
 * 0.5, 1.5), times one ue8m0 scale byte per 128 consecutive elements along the reduction
 * axis (2 + 8/128 = 2.0625 bits per weight).  The E routed experts, contiguous per matrix:
 *   gate_codes, up_codes  [E][f][d/4]   gate_scales, up_scales  [E][f][d/128]
 *   down_codes            [E][d][f/4]   down_scales             [E][d][f/128]
 * All six arrays 16-byte aligned. */
typedef struct {
  const uint8_t* gate_codes;
  const uint8_t* gate_scales;
  const uint8_t* up_codes;
  const uint8_t* up_scales;
  const uint8_t* down_codes;
  const uint8_t* down_scales;
} moe_q2_experts_t;

/* moe_forward for one token (T = 1) with 2-bit routed experts: the routed experts come
 * from `q2` (the same E, d, f as `w`), the shared expert from `w` (FP4, index E; w's
 * routed experts are not read).  Outputs, workspace and rules as for moe_forward at T = 1,
 * in ONE cooperative kernel: the routed experts' units stream the 2-bit codes (decoded to
 * e4m3 in registers, mma.sync e4m3 x e4m3 with fp32 sums per 128-element chunk, then the
 * chunk's weight scale and the token's activation scale), the shared expert's the FP4
 * codes.  d and f multiples of 2048; k <= 32; the shape must fit the single-token kernel
 * (MOE_ERR_INVALID_ARG otherwise). */
int moe_forward_q2(const float* scores, const uint16_t* x_bf16, int k, const moe_weights_t* w,
                   const moe_q2_experts_t* q2, int32_t* topk_idx, float* topk_w,
                   int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                   float* y_routed, float* y_shared, float* out, void* ws, size_t ws_bytes,
                   void* stream);

/* FP8 x FP8 GEMM (NEXT-3): the pages' fp8_gemm beside fp4_gemm ([P1] "补齐软件栈缺失":
 * FP8 activations times FP8 weights, the format of the model's non-FP4 linears).  The
 * page gives no scale layout; read here as e4m3 weights with one fp32 scale per 128 x 128
 * block (rows x reduction) and e4m3 activations with one fp32 scale per row and 128-block
 * (moe_act_quant's codes):
 *   C[m][n] = sum_kb sa[m][kb] * sb[n/128][kb] * sum_{k in block kb} A[m][k] * B[n][k].
 *   A [M][K] e4m3 codes (16-byte aligned), sa [M][K/128] fp32; B [N][K] e4m3 codes
 *   (16-byte aligned), sb [N/128][K/128] fp32; C [M][N] fp32 out (8-byte aligned).
 *   ws: at least moe_fp8_gemm_workspace_size(M, N, K) bytes, 256-byte aligned, contents
 *   need not be initialised (the call clears what it needs).
 * 0 <= M <= 64 (a decode-sized batch: one weight read serves every row of A); N % 128 == 0;
 * K % 512 == 0.  Reads B once (mma.sync e4m3 on the codes, 128-element sums in the tensor
 * core, scales applied in fp32, per-row-block partials added in reduction order). */
size_t moe_fp8_gemm_workspace_size(int M, int N, int K);
int moe_fp8_gemm(const uint8_t* A, const float* sa, int M, int K, const uint8_t* B,
                 const float* sb, int N, float* C, void* ws, size_t ws_bytes, void* stream);

/* An FP8-weight expert (NEXT-3: the real model's shared expert is FP8, not FP4):
 *   gate, up [f][d] e4m3, gate_scales, up_scales [f/128][d/128] fp32;
 *   down [d][f] e4m3, down_scales [d/128][f/128] fp32.  Code arrays 16-byte aligned. */
typedef struct {
  const uint8_t* gate;
  const float* gate_scales;
  const uint8_t* up;
  const float* up_scales;
  const uint8_t* down;
  const float* down_scales;
  int d;
  int f;
} moe_fp8_expert_t;

/* The shared expert with FP8 weights for T tokens: x quantised as in moe_act_quant, then
 * h = silu(g) * u with g, u from one fused FP8 GEMM over the gate and up rows, h
 * re-quantised per 128-block (amax / 448, IEEE divide, round to nearest even), and
 * y_shared = W_down h^ by a second FP8 GEMM.
 *   x_bf16 [T][d] bf16 (16-byte aligned); y_shared [T][d] fp32 out (8-byte aligned).
 *   ws: at least moe_shared_expert_fp8_workspace_size(T, d, f) bytes, 256-byte aligned.
 * 0 <= T <= 64; d, f multiples of 512.  Four kernels on the stream. */
size_t moe_shared_expert_fp8_workspace_size(int T, int d, int f);
/* Where moe_shared_expert_fp8 leaves its intermediates in a workspace laid out for
 * (T, d, f), for tests and tools (the pages have no counterpart): byte offsets of
 * off[0] qx [T][d] e4m3, off[1] sx [T][d/128] fp32, off[2] h [T][f] fp32 (silu(g) * u
 * before re-quantisation), off[3] qh [T][f] e4m3, off[4] sh [T][f/128] fp32.
 * MOE_ERR_INVALID_ARG for shapes the call rejects. */
int moe_shared_expert_fp8_offsets(int T, int d, int f, size_t off[5]);
int moe_shared_expert_fp8(const uint16_t* x_bf16, int T, const moe_fp8_expert_t* w,
                          float* y_shared, void* ws, size_t ws_bytes, void* stream);

/* Expert streaming (NEXT-4, one GPU): routed experts that live in host memory
 * ([P1] "DeepSeek-V4-Flash的可能性": routed experts in host RAM, the shared expert and
 * attention resident; [P2] "核心实现一": experts streamed in as they are needed, kept
 * under an LRU share).  The routed experts are in pinned host memory that the device can
 * read (cudaHostAlloc, or cudaHostRegister with cudaHostRegisterMapped; pass the device
 * pointers): the moe_weights_t layout for E experts, [E][...] per matrix, each array
 * 16-byte aligned. */
typedef struct {
  const uint8_t* gate_codes;
  const uint8_t* gate_scales;
  const uint8_t* up_codes;
  const uint8_t* up_scales;
  const uint8_t* down_codes;
  const uint8_t* down_scales;
} moe_host_experts_t;

/* The HBM expert cache, device memory owned by the caller:
 *   slots      moe_weights_t of S + 1 expert slots (slots.E = S): slots 0..S-1 hold
 *              routed experts, slot S the shared expert (the caller fills it once);
 *   slot_of    [E] int32: slot of each routed expert, -1 when not resident;
 *   expert_of  [S] int32: expert in each slot, -1 when empty;
 *   last_use   [S] int64: step of each slot's last use;
 *   clock      [1] int64: steps so far;
 *   fetch      [1 + 2*32] int32 scratch: this step's fills (count, then expert, slot);
 *   stats      [2] int64: hits and misses accumulated.
 * E routed experts; k <= S. */
typedef struct {
  moe_weights_t slots;
  int32_t* slot_of;
  int32_t* expert_of;
  int64_t* last_use;
  int64_t* clock;
  int32_t* fetch;
  int64_t* stats;
  int E;
} moe_expert_cache_t;

/* Empty cache: slot_of and expert_of to -1, last_use, clock and stats to 0 (enqueued). */
int moe_expert_cache_reset(const moe_expert_cache_t* c, void* stream);

/* moe_forward for one token with the routed experts streamed from `host` through the
 * cache: the top-k of the scores (into topk_idx, topk_w), the cache's LRU step (the
 * selected experts, ascending id, are marked used; each missing one takes the least
 * recently used slot not holding an expert of this token, empty slots first, ties to the
 * lower slot; its expert is evicted), the copy of the missing experts from host memory
 * into their slots (a kernel reading the host arrays over PCIe), then the single-token
 * layer kernel on the slots.  Outputs, workspace (moe_workspace_size(1, k, c->E, d, f))
 * and rules as moe_forward at T = 1; results equal moe_forward's on resident weights bit
 * for bit.  Everything is enqueued on `stream`; the host never waits. */
int moe_forward_streamed(const float* scores, const uint16_t* x_bf16, int k,
                         const moe_host_experts_t* host, const moe_expert_cache_t* c,
                         int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                         int32_t* perm, int32_t* pos, float* y_routed, float* y_shared,
                         float* out, void* ws, size_t ws_bytes, void* stream);

/* Step 8 — combine: out[t][m] = y_shared[t][m] + sum_{j<k} topk_w[t][j] *
 * y_routed[pos[t*k+j]][m], summed in fixed j order in fp32.
 *   y_routed [T*k][d], y_shared [T][d], topk_w [T][k], pos [T*k], out [T][d] fp32.
 * d % 4 == 0; y_routed, y_shared and out 16-byte aligned. */
int moe_combine(const float* y_routed, const float* y_shared, const float* topk_w,
                const int32_t* pos, int T, int k, int d, float* out, void* stream);

/* Bytes of scratch the multi-CTA dispatch uses for T*k pairs over E experts (0 when a
 * batch that small runs the one-CTA form, or on invalid sizes). */
size_t moe_dispatch_workspace_size(int T, int k, int E);

/* Bytes of workspace moe_expert_ffn needs (0 on invalid sizes). */
size_t moe_workspace_size(int T, int k, int E, int d, int f);

/* Where moe_expert_ffn leaves its intermediate results inside a workspace laid out for
 * (T, k, E, d, f): byte offsets from the workspace start, for tests and tools that
 * inspect them.  The pages have no counterpart.  Rows r < T*k are the routed pairs in
 * expert-sorted order (row r = pair perm[r]); row T*k + t is token t's shared-expert row.
 *   off[0] qx [rows][d]     e4m3 codes of the FFN's input rows (the single-token path
 *                           writes row 0 only: the token)
 *   off[1] sx [rows][d/128] fp32 scales of qx
 *   off[2] qh [rows][f]     e4m3 codes of the re-quantised hidden state
 *   off[3] sh [rows][f/128] fp32 scales of qh
 *   off[4] h  [rows][f]     fp32 hidden state before re-quantisation; only the
 *                           single-token path keeps it (SIZE_MAX otherwise)
 * The contents are valid after moe_expert_ffn (or moe_forward) completes on the stream.
 * Returns MOE_OK, or MOE_ERR_INVALID_ARG for sizes moe_workspace_size rejects. */
int moe_workspace_offsets(int T, int k, int E, int d, int f, size_t off[5]);

/* Thread-local message for the last error on this thread ("" if none). */
const char* moe_last_error(void);

/* Upper bound, in nanoseconds of the GPU's global timer, on every device-side wait
 * (mbarrier / pipeline waits in the FFN kernels).  A wait that runs out makes the
 * kernel record MOE_ERR_TIMEOUT, release what it holds and return.  Default 2e9
 * (2 s).  n <= 0 restores the default.  Applies to launches made after the call. */
int moe_set_wait_limit_ns(long long n);

/* Largest batch T that runs the expert FFN as FP4 GEMV kernels (CUDA-core e2m1 decode,
 * mma.sync; the decode paths) instead of the tcgen05 tile kernels: T = 1 the single-token
 * kernels, 2 <= T <= 64 the batched GEMV (groups of up to 8 tokens per expert).  The
 * pages have no counterpart: it is a switch between implementations of the same calls.
 * 0 sends every batch to the tile kernels; values above 64 act as 64.  The GEMV paths
 * also need d and f multiples of 512 and 16-byte aligned scale arrays (the single-token
 * kernel also k + 1 <= the SM count); other shapes take the tile kernels.  Default 64.
 * Applies to calls made after it. */
int moe_set_gemv_max_tokens(int t);

/* Which form of the single-token layer kernel moe_forward (T = 1) and
 * moe_forward_streamed run; the pages have no counterpart (tcti.cn post, "DeepSeek-V4-
 * Flash的可能性": decode is bound by reading the selected experts' weights; both forms
 * read each weight byte once and compute the same layer).  0 (the default): on the CUDA
 * cores (e2m1 decoded to f16 in registers, mma.sync), the faster form on a B200 at the
 * decode sizes.  1: on the tensor cores (tcgen05.mma kind::mxf8f6f4.block_scale on the
 * FP4 codes, unpacked by TMA) where the shapes allow it: d and f multiples of 256 and at
 * most 4096, f such that three experts' h tiles fit in shared memory, k <= 32; other
 * shapes stay on the CUDA cores.  Results of the two forms agree within the
 * floating-point bounds of the parity rules, not bit for bit (their fp32 sums run in
 * different orders); each form is deterministic.  Returns MOE_ERR_INVALID_ARG for other
 * values.  Applies to calls made after it. */
int moe_set_decode_engine(int engine);

/* Testing knob; the pages have no counterpart.  While on, every launch of the
 * single-token FFN kernels makes warp 0 of CTA 0 wait, before its first weight stage, on
 * a shared-memory barrier that nothing completes, so that the wait's time limit
 * (moe_set_wait_limit_ns) runs out: the kernel records MOE_ERR_TIMEOUT in the status word,
 * lets the copies it issued land and returns, and the outputs of that call are
 * incomplete.  This exercises the bounded-wait path without any fault.  0 (the default)
 * turns it off.  Applies to launches made after the call. */
int moe_set_test_stall(int on);

/* Which implementation moe_expert_ffn would run for T tokens with these weights on the
 * current device, under the current moe_set_gemv_max_tokens: MOE_PATH_TILES (tcgen05
 * tiles), MOE_PATH_SINGLE (the single-token kernels) or MOE_PATH_BATCHED (the batched
 * GEMV); a negative MOE_ERR_* on invalid arguments.  The pages have no counterpart; tests
 * and tools use it to know which intermediates a workspace holds. */
#define MOE_PATH_TILES 0
#define MOE_PATH_SINGLE 1
#define MOE_PATH_BATCHED 2
int moe_ffn_path(int T, int k, const moe_weights_t* w);

/* The same for moe_forward, under the current moe_set_decode_engine as well: as
 * moe_ffn_path, except MOE_PATH_SINGLE_TC where the single-token layer kernel runs on the
 * tensor cores. */
#define MOE_PATH_SINGLE_TC 3
int moe_forward_path(int T, int k, const moe_weights_t* w);

/* Synchronise `stream`, then return MOE_ERR_CUDA for a pending CUDA error,
 * MOE_ERR_TIMEOUT if a device-side wait expired since the last call (clearing the
 * record), else MOE_OK. */
int moe_sync_status(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* BITMOE_H */
