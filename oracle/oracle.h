/*
 * Oracle for the routed-expert MoE layer — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar C implementation of what the hot path computes, used by
 * the tests, by smoke() and by the benchmark's CPU-baseline leg to check the
 * CUDA library.  Nothing on the product path may link or call it.  It shares no
 * code with the CUDA library.
 *
 * Sources (the pages' titles; sections as the pages name them):
 *  - "DeepSeek-V4-Flash on 4x RTX 2080 Ti" forum post (tcti.cn), section
 *    "DeepSeek-V4-Flash的可能性": routed experts are FP4, top-6 of 256 per token,
 *    an always-on shared expert sits beside them; section "补齐软件栈缺失":
 *    act_quant feeds FP8-quantised activations to fp4_gemm (FP8 act x FP4 packed
 *    weight).
 *  - "deepseek-v4-flash-0731-in-c" article (dpshk.com), section
 *    "核心实现三：多 token 批处理" (an expert's weights are read once for all tokens
 *    routed to it) and "核心实现四：低比特融合算子" (FP4 dequantised inside the
 *    GEMV, gate and up share one quantised input).
 *  - What those pages leave open (d, f, block sizes, scale formats, gating) is
 *    fixed as: e2m1 codes packed two per byte (low nibble = even element), one
 *    ue8m0 scale per 32 consecutive elements along the reduction axis,
 *    activations quantised per 128-element block to e4m3 with scale amax/448 in
 *    fp32, combine weight = sigmoid of the selected scores renormalised to 1,
 *    shared expert added with weight 1.
 *  Formats: OCP Microscaling Formats (MX) Specification v1.0 (e2m1, e4m3, e8m0).
 *  - "一張 22G 老卡跑 284B" post (ai-muninn.com): the routed experts of the deployed model
 *    are 2-bit (IQ2_XXS, 2.0625 bits per weight) while the always-resident weights
 *    (shared expert included) stay at higher precision; the "2-bit routed experts only"
 *    of the ds4 engine (smzdm.com post) is the same split.  The pages name the bit rate,
 *    not the code book, so the 2-bit codec here is read as: four 2-bit codes per byte
 *    (element i of a byte in bits 2i..2i+1), value = code - 1.5 (the uniform
 *    four-level grid -1.5, -0.5, 0.5, 1.5), times one ue8m0 scale per 128 consecutive
 *    elements along the reduction axis: 2 + 8/128 = 2.0625 bits per weight.
 *  - tcti.cn post, section "补齐软件栈缺失": fp8_gemm (FP8 activation x FP8 weight) for the
 *    model's FP8 linears; the SURVEY's NEXT-3 reads the shared expert as one of them.  The
 *    page gives no scale layout; read here as e4m3 weights with one fp32 scale per
 *    128 x 128 block (rows x reduction) and activations quantised per token and 128-block
 *    exactly as for the FP4 path.
 *
 * Floating point: all sums are in double.  Activation quantisation is done in
 * fp32 arithmetic (divide, then round to nearest e4m3, ties to even mantissa,
 * saturating at +-448) because that is how the quantised codes are defined.
 */
#ifndef BITMOE_ORACLE_H
#define BITMOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Per-expert weight pointers.  gate/up: rows = f, K = d.  down: rows = d, K = f.
 * codec ORACLE_FP4: codes [rows][K/2] bytes, scales [rows][K/32] bytes.
 * codec ORACLE_Q2:  codes [rows][K/4] bytes, scales [rows][K/128] bytes.
 * codec ORACLE_FP8: codes [rows][K] e4m3 bytes; the scales pointer points to fp32 values
 *                   [rows/128][K/128] (one per 128 x 128 block). */
#define ORACLE_FP4 0
#define ORACLE_Q2 1
#define ORACLE_FP8 2
typedef struct {
    const uint8_t* gate_codes;
    const uint8_t* gate_scales;
    const uint8_t* up_codes;
    const uint8_t* up_scales;
    const uint8_t* down_codes;
    const uint8_t* down_scales;
    int codec;
} oracle_expert_t;

/* Format decoding from bit fields (OCP MX v1.0). */
double oracle_e2m1_value(int code);   /* code in [0,16) */
double oracle_e4m3_value(int code);   /* code in [0,256); NaN for 0x7F/0xFF */
double oracle_ue8m0_value(int code);  /* code in [0,256); NaN for 0xFF */
double oracle_q2_value(int code);     /* code in [0,4): code - 1.5 */

/* fp32 -> e4m3fn code: round to nearest, ties to even mantissa, saturate to +-448. */
uint8_t oracle_e4m3_encode(float v);

/* Quantise n (multiple of 128) fp32 values per 128-block: s = amax/448 (fp32),
 * s = 1 when amax == 0, q = e4m3(v / s). */
void oracle_quant_blocks(const float* v, int n, uint8_t* q, float* s);

/* bf16 activations [T][d] -> e4m3 codes [T][d], fp32 scales [T][d/128]. */
void oracle_act_quant(const uint16_t* x_bf16, int T, int d, uint8_t* q, float* s);

/* Router scores: scores[t][e] = sum_i x[t][i] * W_router[e][i] over bf16 x [T][d] and
 * W_router [E][d], in double.  (dpshk.com article, "核心实现一": the router picks each
 * token's experts.)  The selection is oracle_route_topk on these scores rounded to fp32. */
void oracle_router_scores(const uint16_t* x_bf16, const uint16_t* w_bf16, int T, int d, int E,
                          double* scores);

/* Top-k routing: k largest scores per token, descending, ties to the lower expert
 * index; w_j = sigmoid(s_j) / sum_j' sigmoid(s_j') in double. */
void oracle_route_topk(const float* scores, int T, int E, int k, int32_t* idx, double* w);

/* Stable grouping of the T*k (token, slot) pairs by expert. */
void oracle_dispatch(const int32_t* idx, int T, int k, int E, int32_t* counts,
                     int32_t* offsets, int32_t* perm, int32_t* pos);

/* out[r] = sum_k W[r,k] * xhat[k] for `rows` rows of an FP4 matrix with K columns,
 * W[r,k] = e2m1(code) * ue8m0(scale[r, k/32]), in double. */
void oracle_fp4_gemv(const uint8_t* codes, const uint8_t* scales, int rows, int K,
                     const double* xhat, double* out);

/* The same for a 2-bit matrix: W[r,k] = q2(code) * ue8m0(scale[r, k/128]), code of
 * element k in bits 2(k%4)..2(k%4)+1 of byte codes[r, k/4]; in double. */
void oracle_q2_gemv(const uint8_t* codes, const uint8_t* scales, int rows, int K,
                    const double* xhat, double* out);

/* fp8_gemm: C[m][n] = sum_k (e4m3(A[m,k]) * sa[m, k/128]) * (e4m3(B[n,k]) * sb[n/128, k/128])
 * in double; A [M][K] and B [N][K] e4m3 codes, sa [M][K/128], sb [N/128][K/128] fp32,
 * C [M][N].  K and N multiples of 128. */
void oracle_fp8_gemm(const uint8_t* A, const float* sa, int M, const uint8_t* B,
                     const float* sb, int N, int K, double* C);

/* One expert FFN over a group of ntok tokens that share its weights (layer-major:
 * each weight row is decoded once and dotted with every token of the group).
 * qx [ntok][d] e4m3 codes, sx [ntok][d/128]; y [ntok][d] double out.
 * Optional h_q/h_s (may be NULL) receive the re-quantised hidden state
 * [ntok][f] codes and [ntok][f/128] scales. */
void oracle_expert_ffn(const oracle_expert_t* w, int d, int f, const uint8_t* qx,
                       const float* sx, int ntok, double* y, uint8_t* h_q, float* h_s);
/* Same, also returning the fp32 hidden state before re-quantisation (h_f32 [ntok][f],
 * may be NULL). */
void oracle_expert_ffn_h(const oracle_expert_t* w, int d, int f, const uint8_t* qx,
                         const float* sx, int ntok, double* y, uint8_t* h_q, float* h_s,
                         float* h_f32);

/* Weighted combine for one token: out[m] = ysh[m] + sum_j w[j] * y[j][m]. */
void oracle_combine_token(const double* ysh, const double* y, const double* w, int k, int d,
                          double* out);

/* Layer output for a selection of tokens.  experts[0..E] (index E = shared) may be
 * NULL for experts none of the selected tokens uses.  x_bf16 [T][d]; idx [T][k];
 * w [T][k].  For each of the nsel tokens tok[i]: y_pair [nsel][k][d], y_sh [nsel][d],
 * out [nsel][d]. */
void oracle_moe_tokens(const uint16_t* x_bf16, int T, int d, int f, int E, int k,
                       const oracle_expert_t* experts, const int32_t* idx, const double* w,
                       const int32_t* tok, int nsel, double* y_pair, double* y_sh, double* out);

/* Whole layer, layer-major (every expert with a non-empty group runs once over its
 * group).  Outputs y_pair [T*k][d] (pair order t*k+j), y_sh [T][d], out [T][d]. */
void oracle_moe_layer(const uint16_t* x_bf16, int T, int d, int f, int E, int k,
                      const oracle_expert_t* experts, const int32_t* idx, const double* w,
                      double* y_pair, double* y_sh, double* out);

void oracle_set_threads(int n);
int oracle_get_threads(void);

#ifdef __cplusplus
}
#endif
#endif
