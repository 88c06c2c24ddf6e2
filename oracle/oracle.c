/*
 * Oracle for the routed-expert MoE layer — TEST INFRASTRUCTURE ONLY.
 * See oracle.h for the sources followed and the numeric contract.
 * Plain scalar C99, double accumulation, OpenMP over independent rows/tokens.
 * Built with -ffp-contract=off so fp32 steps round exactly as written.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------------------
 * Formats (OCP MX v1.0): values are built from the bit fields of each code.
 * ------------------------------------------------------------------------- */

/* e2m1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent 0 is subnormal. */
double oracle_e2m1_value(int code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? ldexp((double)m, -1) : ldexp(1.0 + m / 2.0, e - 1);
    return s ? -v : v;
}

/* e4m3fn: 1 sign, 4 exponent (bias 7), 3 mantissa bits; S.1111.111 is NaN, no inf. */
double oracle_e4m3_value(int code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* e8m0 (unsigned): 2^(b - 127); 0xFF is NaN. */
double oracle_ue8m0_value(int code) {
    if ((code & 0xFF) == 0xFF) return NAN;
    return ldexp(1.0, (code & 0xFF) - 127);
}

/* Round to nearest integer, ties to even (exact for the small magnitudes used). */
static double rint_even(double a) {
    double fl = floor(a), diff = a - fl;
    if (diff > 0.5) return fl + 1.0;
    if (diff < 0.5) return fl;
    return fmod(fl, 2.0) == 0.0 ? fl : fl + 1.0;
}

/* fp32 -> e4m3fn with round-to-nearest-even and saturation to +-448 (satfinite).
 * |v| < 2^-6 is in the subnormal range (step 2^-9); otherwise the step within
 * the binade [2^e, 2^(e+1)) is 2^(e-3). */
uint8_t oracle_e4m3_encode(float v) {
    double a = fabs((double)v);
    uint8_t sign = (v < 0.0f || (v == 0.0f && signbit(v))) ? 0x80 : 0x00;
    if (isnan(v)) return 0x7F;
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        double m = rint_even(a / ldexp(1.0, -9));         /* 0..8 */
        if (m >= 8.0) return (uint8_t)(sign | 0x08);      /* rounds up to 2^-6 */
        return (uint8_t)(sign | (uint8_t)m);
    }
    int e = (int)floor(log2(a));
    if (ldexp(1.0, e) > a) e -= 1;                         /* guard log2 rounding */
    if (ldexp(1.0, e + 1) <= a) e += 1;
    double r = rint_even(a / ldexp(1.0, e - 3));          /* 8..16 */
    if (r >= 16.0) { e += 1; r = 8.0; }
    if (e > 8 || (e == 8 && r > 14.0)) return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | ((int)r - 8)));
}

static inline float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Per-128-block activation quantisation in fp32 (tcti.cn post, "补齐软件栈缺失":
 * act_quant provides the FP8 activations of the FP4 linears). */
void oracle_quant_blocks(const float* v, int n, uint8_t* q, float* s) {
    for (int b = 0; b < n / 128; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 128; ++i) {
            float a = fabsf(v[b * 128 + i]);
            if (a > amax) amax = a;
        }
        volatile float sc = amax / 448.0f;          /* IEEE fp32 divide */
        if (amax == 0.0f) sc = 1.0f;
        s[b] = sc;
        for (int i = 0; i < 128; ++i) {
            volatile float t = v[b * 128 + i] / sc;  /* fp32 quotient, then e4m3 RNE */
            q[b * 128 + i] = oracle_e4m3_encode(t);
        }
    }
}

void oracle_act_quant(const uint16_t* x_bf16, int T, int d, uint8_t* q, float* s) {
    float* row = (float*)malloc(sizeof(float) * (size_t)d);
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < d; ++i) row[i] = bf16_to_f32(x_bf16[(size_t)t * d + i]);
        oracle_quant_blocks(row, d, q + (size_t)t * d, s + (size_t)t * (d / 128));
    }
    free(row);
}

/* ---------------------------------------------------------------------------
 * Routing (tcti.cn post, "DeepSeek-V4-Flash的可能性": top-6 of the routed experts
 * per token): rank all experts by (score descending, index ascending), keep k.
 * ------------------------------------------------------------------------- */
static int rank_before(float sa, int ia, float sb, int ib) {
    if (sa != sb) return sa > sb;
    return ia < ib;
}

/* Router scores (dpshk.com article, "核心实现一": the router decides each token's experts
 * from its hidden state): scores[t][e] = sum_i x[t][i] * W[e][i] over the bf16 inputs,
 * summed in double (every product of two bf16 values is exact in double). */
void oracle_router_scores(const uint16_t* x_bf16, const uint16_t* w_bf16, int T, int d, int E,
                          double* scores) {
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += (double)bf16_to_f32(x_bf16[(size_t)t * d + i]) *
                       (double)bf16_to_f32(w_bf16[(size_t)e * d + i]);
            scores[(size_t)t * E + e] = acc;
        }
}

void oracle_route_topk(const float* scores, int T, int E, int k, int32_t* idx, double* w) {
    int* order = (int*)malloc(sizeof(int) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        const float* s = scores + (size_t)t * E;
        for (int e = 0; e < E; ++e) order[e] = e;
        /* full insertion sort by the ranking key: plain and obviously correct */
        for (int i = 1; i < E; ++i) {
            int cur = order[i], j = i - 1;
            while (j >= 0 && rank_before(s[cur], cur, s[order[j]], order[j])) {
                order[j + 1] = order[j];
                --j;
            }
            order[j + 1] = cur;
        }
        double sum = 0.0;
        for (int j = 0; j < k; ++j) {
            idx[(size_t)t * k + j] = order[j];
            sum += 1.0 / (1.0 + exp(-(double)s[order[j]]));
        }
        for (int j = 0; j < k; ++j)
            w[(size_t)t * k + j] = (1.0 / (1.0 + exp(-(double)s[order[j]]))) / sum;
    }
    free(order);
}

/* ---------------------------------------------------------------------------
 * Dispatch (dpshk.com article, "核心实现三：多 token 批处理": group the tokens by
 * expert so that each expert is read once for its whole group).  Pairs are the
 * flat ids t*k + j; within an expert they keep ascending id order (stable).
 * ------------------------------------------------------------------------- */
void oracle_dispatch(const int32_t* idx, int T, int k, int E, int32_t* counts,
                     int32_t* offsets, int32_t* perm, int32_t* pos) {
    int P = T * k, p = 0;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        int c = 0;
        for (int i = 0; i < P; ++i) {
            if (idx[i] == e) {
                perm[p] = i;
                pos[i] = p;
                ++p;
                ++c;
            }
        }
        counts[e] = c;
        offsets[e + 1] = offsets[e] + c;
    }
}

/* ---------------------------------------------------------------------------
 * Fused low-bit GEMV (dpshk.com article, "核心实现四：低比特融合算子"): each FP4
 * weight is decoded inside the dot product; no float copy of the matrix.
 * ------------------------------------------------------------------------- */
static inline double fp4_weight(const uint8_t* codes, const uint8_t* scales, int K, int r,
                                int c) {
    uint8_t byte = codes[(size_t)r * (K / 2) + c / 2];
    int code = (c & 1) ? (byte >> 4) : (byte & 0x0F);
    return oracle_e2m1_value(code) * oracle_ue8m0_value(scales[(size_t)r * (K / 32) + c / 32]);
}

/* 2-bit routed-expert codec (ai-muninn.com post "一張 22G 老卡跑 284B": IQ2_XXS routed
 * experts at 2.0625 bits per weight; the code book is this library's reading, see
 * oracle.h): value = code - 1.5, one ue8m0 scale per 128 elements. */
double oracle_q2_value(int code) { return (double)(code & 3) - 1.5; }

static inline double q2_weight(const uint8_t* codes, const uint8_t* scales, int K, int r,
                               int c) {
    uint8_t byte = codes[(size_t)r * (K / 4) + c / 4];
    int code = (byte >> (2 * (c & 3))) & 3;
    return oracle_q2_value(code) * oracle_ue8m0_value(scales[(size_t)r * (K / 128) + c / 128]);
}

static int g_threads = 1;
void oracle_set_threads(int n) { g_threads = n < 1 ? 1 : n; }
int oracle_get_threads(void) { return g_threads; }

void oracle_fp4_gemv(const uint8_t* codes, const uint8_t* scales, int rows, int K,
                     const double* xhat, double* out) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int c = 0; c < K; ++c) acc += fp4_weight(codes, scales, K, r, c) * xhat[c];
        out[r] = acc;
    }
}

/* FP8 weights (tcti.cn post, "补齐软件栈缺失": fp8_gemm): e4m3 codes, one fp32 scale per
 * 128 x 128 block. */
static inline double fp8_weight(const uint8_t* codes, const uint8_t* scales, int K, int r,
                                int c) {
    const float* s = (const float*)scales;
    return oracle_e4m3_value(codes[(size_t)r * K + c]) *
           (double)s[(size_t)(r / 128) * (K / 128) + c / 128];
}

void oracle_fp8_gemm(const uint8_t* A, const float* sa, int M, const uint8_t* B,
                     const float* sb, int N, int K, double* C) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int n = 0; n < N; ++n) {
        for (int m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += oracle_e4m3_value(A[(size_t)m * K + k]) * (double)sa[(size_t)m * (K / 128) + k / 128] *
                       fp8_weight(B, (const uint8_t*)sb, K, n, k);
            C[(size_t)m * N + n] = acc;
        }
    }
}

void oracle_q2_gemv(const uint8_t* codes, const uint8_t* scales, int rows, int K,
                    const double* xhat, double* out) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int c = 0; c < K; ++c) acc += q2_weight(codes, scales, K, r, c) * xhat[c];
        out[r] = acc;
    }
}

/* Decode one weight row (FP4 or 2-bit codec) into doubles. */
static void decode_row(int codec, const uint8_t* codes, const uint8_t* scales, int K, int r,
                       double* dst) {
    for (int c = 0; c < K; ++c)
        dst[c] = codec == ORACLE_Q2 ? q2_weight(codes, scales, K, r, c)
                 : codec == ORACLE_FP8 ? fp8_weight(codes, scales, K, r, c)
                                       : fp4_weight(codes, scales, K, r, c);
}

/* One expert over a group of tokens: g = Wg xhat, u = Wu xhat, h = silu(g) * u
 * rounded to fp32 and re-quantised per 128 as the activations were, y = Wd hhat.
 * Each weight row is decoded once and used for every token of the group. */
void oracle_expert_ffn(const oracle_expert_t* w, int d, int f, const uint8_t* qx,
                       const float* sx, int ntok, double* y, uint8_t* h_q, float* h_s) {
    oracle_expert_ffn_h(w, d, f, qx, sx, ntok, y, h_q, h_s, NULL);
}

void oracle_expert_ffn_h(const oracle_expert_t* w, int d, int f, const uint8_t* qx,
                         const float* sx, int ntok, double* y, uint8_t* h_q, float* h_s,
                         float* h_f32) {
    double* xhat = (double*)malloc(sizeof(double) * (size_t)ntok * d);
    double* g = (double*)malloc(sizeof(double) * (size_t)ntok * f);
    double* u = (double*)malloc(sizeof(double) * (size_t)ntok * f);
    float* h = (float*)malloc(sizeof(float) * (size_t)ntok * f);
    uint8_t* hq = (uint8_t*)malloc((size_t)ntok * f);
    float* hs = (float*)malloc(sizeof(float) * (size_t)ntok * (f / 128));
    double* hhat = (double*)malloc(sizeof(double) * (size_t)ntok * f);

    for (int t = 0; t < ntok; ++t)
        for (int c = 0; c < d; ++c)
            xhat[(size_t)t * d + c] = oracle_e4m3_value(qx[(size_t)t * d + c]) *
                                      (double)sx[(size_t)t * (d / 128) + c / 128];

#pragma omp parallel num_threads(g_threads)
    {
        double* rg = (double*)malloc(sizeof(double) * (size_t)d);
        double* ru = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
        for (int n = 0; n < f; ++n) {
            decode_row(w->codec, w->gate_codes, w->gate_scales, d, n, rg);
            decode_row(w->codec, w->up_codes, w->up_scales, d, n, ru);
            for (int t = 0; t < ntok; ++t) {
                const double* xt = xhat + (size_t)t * d;
                double ag = 0.0, au = 0.0;
                for (int c = 0; c < d; ++c) {
                    ag += rg[c] * xt[c];
                    au += ru[c] * xt[c];
                }
                g[(size_t)t * f + n] = ag;
                u[(size_t)t * f + n] = au;
            }
        }
        free(rg);
        free(ru);
    }

    /* SwiGLU in double, rounded to fp32, then per-128 e4m3 re-quantisation */
    for (int t = 0; t < ntok; ++t) {
        for (int n = 0; n < f; ++n) {
            double gv = g[(size_t)t * f + n];
            double hv = gv / (1.0 + exp(-gv)) * u[(size_t)t * f + n];
            h[(size_t)t * f + n] = (float)hv;
        }
        oracle_quant_blocks(h + (size_t)t * f, f, hq + (size_t)t * f, hs + (size_t)t * (f / 128));
        for (int n = 0; n < f; ++n)
            hhat[(size_t)t * f + n] = oracle_e4m3_value(hq[(size_t)t * f + n]) *
                                      (double)hs[(size_t)t * (f / 128) + n / 128];
    }
    if (h_f32) memcpy(h_f32, h, sizeof(float) * (size_t)ntok * f);
    if (h_q) memcpy(h_q, hq, (size_t)ntok * f);
    if (h_s) memcpy(h_s, hs, sizeof(float) * (size_t)ntok * (f / 128));

#pragma omp parallel num_threads(g_threads)
    {
        double* rd = (double*)malloc(sizeof(double) * (size_t)f);
#pragma omp for schedule(static)
        for (int m = 0; m < d; ++m) {
            decode_row(w->codec, w->down_codes, w->down_scales, f, m, rd);
            for (int t = 0; t < ntok; ++t) {
                const double* ht = hhat + (size_t)t * f;
                double acc = 0.0;
                for (int n = 0; n < f; ++n) acc += rd[n] * ht[n];
                y[(size_t)t * d + m] = acc;
            }
        }
        free(rd);
    }
    free(xhat); free(g); free(u); free(h); free(hq); free(hs); free(hhat);
}

/* Routing-weighted combine; the shared expert is added with weight 1. */
void oracle_combine_token(const double* ysh, const double* y, const double* w, int k, int d,
                          double* out) {
    for (int m = 0; m < d; ++m) {
        double acc = ysh[m];
        for (int j = 0; j < k; ++j) acc += w[j] * y[(size_t)j * d + m];
        out[m] = acc;
    }
}

void oracle_moe_tokens(const uint16_t* x_bf16, int T, int d, int f, int E, int k,
                       const oracle_expert_t* experts, const int32_t* idx, const double* w,
                       const int32_t* tok, int nsel, double* y_pair, double* y_sh, double* out) {
    (void)T;
    uint8_t* q = (uint8_t*)malloc((size_t)d);
    float* s = (float*)malloc(sizeof(float) * (size_t)(d / 128));
    for (int i = 0; i < nsel; ++i) {
        int t = tok[i];
        oracle_act_quant(x_bf16 + (size_t)t * d, 1, d, q, s);
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            oracle_expert_ffn(&experts[e], d, f, q, s, 1, y_pair + ((size_t)i * k + j) * d,
                              NULL, NULL);
        }
        oracle_expert_ffn(&experts[E], d, f, q, s, 1, y_sh + (size_t)i * d, NULL, NULL);
        oracle_combine_token(y_sh + (size_t)i * d, y_pair + (size_t)i * k * d,
                             w + (size_t)t * k, k, d, out + (size_t)i * d);
    }
    free(q);
    free(s);
}

void oracle_moe_layer(const uint16_t* x_bf16, int T, int d, int f, int E, int k,
                      const oracle_expert_t* experts, const int32_t* idx, const double* w,
                      double* y_pair, double* y_sh, double* out) {
    int P = T * k;
    uint8_t* qx = (uint8_t*)malloc((size_t)T * d);
    float* sx = (float*)malloc(sizeof(float) * (size_t)T * (d / 128));
    oracle_act_quant(x_bf16, T, d, qx, sx);

    int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1));
    int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1));
    oracle_dispatch(idx, T, k, E, counts, offsets, perm, pos);

    /* layer-major: each routed expert once over its whole group */
    for (int e = 0; e < E; ++e) {
        int n = counts[e];
        if (n == 0) continue;
        uint8_t* gq = (uint8_t*)malloc((size_t)n * d);
        float* gs = (float*)malloc(sizeof(float) * (size_t)n * (d / 128));
        double* gy = (double*)malloc(sizeof(double) * (size_t)n * d);
        for (int i = 0; i < n; ++i) {
            int t = perm[offsets[e] + i] / k;
            memcpy(gq + (size_t)i * d, qx + (size_t)t * d, (size_t)d);
            memcpy(gs + (size_t)i * (d / 128), sx + (size_t)t * (d / 128),
                   sizeof(float) * (size_t)(d / 128));
        }
        oracle_expert_ffn(&experts[e], d, f, gq, gs, n, gy, NULL, NULL);
        for (int i = 0; i < n; ++i)
            memcpy(y_pair + (size_t)perm[offsets[e] + i] * d, gy + (size_t)i * d,
                   sizeof(double) * (size_t)d);
        free(gq); free(gs); free(gy);
    }
    /* shared expert over all tokens */
    if (T > 0) oracle_expert_ffn(&experts[E], d, f, qx, sx, T, y_sh, NULL, NULL);
    for (int t = 0; t < T; ++t)
        oracle_combine_token(y_sh + (size_t)t * d, y_pair + (size_t)t * k * d, w + (size_t)t * k,
                             k, d, out + (size_t)t * d);
    free(qx); free(sx); free(counts); free(offsets); free(perm); free(pos);
}
