/*
 * bitlinear_oracle.c -- plain, slow CPU oracle for the BitLinear W1.58A8 forward
 * of BitNet b1.58.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg load this file's library. The product path (the CUDA
 * library) neither includes, links nor calls anything here, and this file
 * includes nothing from the product. Each function is the step of the method
 * written out as naive loops, in the order the method defines it, with no
 * blocking, fusion or reordering.
 *
 * Sources (pages on BitNet b1.58 2B4T; each function cites the passage it follows):
 *   [card]  "BitNet b1.58 2B4T Technical Report" paper card (ai-papers.xuzou.cn),
 *           sections "Method Adaptation", "Compute Setup", "Bottleneck".
 *   [news]  fishai news digest of the 2B4T report (news.fishai.com.cn/news/3455510),
 *           the list of what a BitLinear layer contains.
 *   [dig]   dignews article on the 2B4T release (dignews.cc), section 2
 *           "core innovations of the architecture".
 *   [wiki]  wikiprompt "1.58-bit large language model", introduction.
 *
 * Readings where the sources above are silent (every one is listed with its reason in the
 * design notes of the repository):
 *   - gamma is one scalar per weight tensor: gamma = mean |W|, summed in fp64 in
 *     row-major order, divided in fp64 by N*K and rounded once to fp32.
 *   - Wq = clip(rint(W / (gamma + 1e-5f)), -1, 1); the division is one IEEE fp32
 *     division and rint rounds half to even.
 *   - s = 127 / max(max_k |x|, 1e-5f) per token (IEEE fp32 division);
 *     xq = clip(rint(x * s), -128, 127) with x * s one fp32 multiply.
 *   - packed byte j of row n holds weights k = 4j..4j+3; weight 4j+i sits in bits
 *     2i..2i+1 as the code q + 1 (0, 1, 2); code 3 is invalid.
 *   - y = bf16_rn(float(acc) * (gamma / s)), optionally
 *     y = bf16_rn(float(residual) + float(acc) * (gamma / s)).
 *   - FFN: g, u dequantised in fp32 (not rounded to bf16); h = (max(g,0)^2) * u;
 *     subln RMSNorm with unit weight: r = 1 / sqrtf(float(sum_j h_j^2 / f) + 1e-5f)
 *     with the sum in fp64; hn = h * r; hn re-quantised per token like x; down
 *     projection dequantised and added to the bf16 residual.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 * -ffp-contract=off keeps every multiply and add a separately rounded IEEE
 * operation, which is what the readings above specify.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_W_EPS 1e-5f   /* eps in W / (gamma + eps) */
#define ORC_X_EPS 1e-5f   /* floor on the per-token absmax */
#define ORC_QB 127.0f     /* int8 activation range: codes in [-128, 127], scale to 127 */
#define ORC_RMS_EPS 1e-5f /* subln RMSNorm eps */

/* Threads of the OpenMP loops over independent output elements (timing only:
 * results do not depend on it). Returns the count now in effect.             */
int orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* bf16 <-> fp32. bf16 is the upper half of an fp32 word; widening is exact and
 * narrowing rounds to nearest, ties to even, keeping NaN a NaN.              */
float orc_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

uint16_t orc_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep = u >> 16;
    uint32_t rest = u & 0xffffu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1u;
    return (uint16_t)keep;
}

void orc_bf16_to_f32_array(const uint16_t* h, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f32(h[i]);
}

void orc_f32_to_bf16_array(const float* f, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(f[i]);
}

/* ------------------------------------------------------------------------- */
/* absmean weight quantisation, [card] "Method Adaptation" (weights quantised to
 * the ternary values {-1, 0, +1} with absmean quantisation in the forward pass),
 * [news] BitLinear list (weight quantisation), [dig] section 2.
 * gamma = mean |W| over the whole tensor.                                      */
float orc_absmean(const float* W, int64_t n) {
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += fabs((double)W[i]);
    return (float)(s / (double)n);
}

/* Wq = clip(rint(W / (gamma + eps)), -1, 1). */
void orc_ternarize(const float* W, int64_t n, float gamma, int8_t* q) {
    float d = gamma + ORC_W_EPS;
    for (int64_t i = 0; i < n; ++i) {
        float r = rintf(W[i] / d);
        if (r > 1.0f) r = 1.0f;
        if (r < -1.0f) r = -1.0f;
        q[i] = (int8_t)r;
    }
}

/* ------------------------------------------------------------------------- */
/* Packing: four ternary weights in one 8-bit value stored in HBM, [card]
 * "Method Adaptation" (pack-store-load-unpack-compute), [dig] section 2.
 * q is [N, K] row-major, Wp is [N, K/4] row-major, K % 4 == 0.                 */
void orc_pack(const int8_t* q, int64_t N, int64_t K, uint8_t* Wp) {
    int64_t KB = K / 4;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < KB; ++j) {
            unsigned b = 0;
            for (int i = 0; i < 4; ++i) {
                unsigned code = (unsigned)(q[n * K + 4 * j + i] + 1);
                b |= code << (2 * i);
            }
            Wp[n * KB + j] = (uint8_t)b;
        }
    }
}

/* Inverse of orc_pack. Returns the number of invalid (== 3) codes; an invalid
 * code decodes to 0 so that the output is defined.                            */
int64_t orc_unpack(const uint8_t* Wp, int64_t N, int64_t K, int8_t* q) {
    int64_t KB = K / 4, bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            unsigned code = ((unsigned)Wp[n * KB + k / 4] >> (2 * (k % 4))) & 3u;
            if (code == 3u) {
                ++bad;
                q[n * K + k] = 0;
            } else {
                q[n * K + k] = (int8_t)((int)code - 1);
            }
        }
    }
    return bad;
}

/* Whole weight path: gamma, ternarise, pack. Wq scratch is allocated here. */
int orc_pack_weights(const float* W, int64_t N, int64_t K, uint8_t* Wp, float* gamma_out) {
    int8_t* q = (int8_t*)malloc((size_t)(N * K));
    if (!q) return -1;
    float gamma = orc_absmean(W, N * K);
    orc_ternarize(W, N * K, gamma, q);
    orc_pack(q, N, K, Wp);
    free(q);
    *gamma_out = gamma;
    return 0;
}

/* ------------------------------------------------------------------------- */
/* absmax per-token activation quantisation to int8, [card] "Method Adaptation"
 * (activations quantised per token with absmax to 8-bit integers), [news]
 * BitLinear list (activation quantisation). x is [M, K] fp32 (bf16 widened).  */
void orc_quant_act(const float* x, int64_t M, int64_t K, int8_t* xq, float* s, int32_t* xsum) {
    for (int64_t m = 0; m < M; ++m) {
        const float* xr = x + m * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(xr[k]);
            if (a > amax) amax = a;
        }
        float sm = ORC_QB / fmaxf(amax, ORC_X_EPS);
        int32_t sum = 0;
        for (int64_t k = 0; k < K; ++k) {
            float r = rintf(xr[k] * sm);
            if (r > 127.0f) r = 127.0f;
            if (r < -128.0f) r = -128.0f;
            xq[m * K + k] = (int8_t)r;
            sum += (int32_t)r;
        }
        s[m] = sm;
        if (xsum) xsum[m] = sum;
    }
}

/* ------------------------------------------------------------------------- */
/* The integer contraction acc[m, n] = sum_k Wq[n, k] * xq[m, k], [card]
 * "Method Adaptation" (the unpacked weights multiplied with the int8
 * activations). Exact in int64, stored as int32 (|acc| <= 127 * K < 2^31).   */
void orc_int_gemm(const int8_t* q, const int8_t* xq, int64_t M, int64_t N, int64_t K, int32_t* acc) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t a = 0;
            for (int64_t k = 0; k < K; ++k) a += (int64_t)q[n * K + k] * (int64_t)xq[m * K + k];
            acc[m * N + n] = (int32_t)a;
        }
    }
}

/* Same contraction reading the packed bytes directly (decode per element). */
void orc_int_gemm_packed(const uint8_t* Wp, const int8_t* xq, int64_t M, int64_t N, int64_t K, int32_t* acc) {
    int64_t KB = K / 4;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t a = 0;
            for (int64_t k = 0; k < K; ++k) {
                int code = (int)(((unsigned)Wp[n * KB + k / 4] >> (2 * (k % 4))) & 3u);
                a += (int64_t)(code - 1) * (int64_t)xq[m * K + k];
            }
            acc[m * N + n] = (int32_t)a;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Dequantisation y = acc * gamma / s (reading: gamma / s as one fp32 division,
 * then one fp32 multiply), optional bf16 residual added in fp32, bf16 output. */
void orc_dequant(const int32_t* acc, float gamma, const float* s, int64_t M, int64_t N,
                 const uint16_t* residual, uint16_t* y, float* y32) {
    for (int64_t m = 0; m < M; ++m) {
        float deq = gamma / s[m];
        for (int64_t n = 0; n < N; ++n) {
            float v = (float)acc[m * N + n] * deq;
            if (residual) v = orc_bf16_to_f32(residual[m * N + n]) + v;
            if (y32) y32[m * N + n] = v;
            y[m * N + n] = orc_f32_to_bf16(v);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* One BitLinear forward, [dig] section 2 (nn.Linear replaced by BitLinear),
 * [card] "Method Adaptation": quantise x per token, contract with the packed
 * ternary weights, dequantise to bf16. No bias ([news], [card]: no bias terms).
 * x, residual and y are bf16 bit patterns. Optional outputs may be NULL.      */
int orc_forward(const uint8_t* Wp, float gamma, int64_t N, int64_t K,
                const uint16_t* x, int64_t M, const uint16_t* residual,
                uint16_t* y, int32_t* acc_out, int8_t* xq_out, float* s_out, int32_t* xsum_out) {
    float* xf = (float*)malloc(sizeof(float) * (size_t)(M * K));
    int8_t* xq = (int8_t*)malloc((size_t)(M * K));
    float* s = (float*)malloc(sizeof(float) * (size_t)M);
    int32_t* xsum = (int32_t*)malloc(sizeof(int32_t) * (size_t)M);
    int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * N));
    if (!xf || !xq || !s || !xsum || !acc) {
        free(xf); free(xq); free(s); free(xsum); free(acc);
        return -1;
    }
    orc_bf16_to_f32_array(x, M * K, xf);
    orc_quant_act(xf, M, K, xq, s, xsum);
    orc_int_gemm_packed(Wp, xq, M, N, K, acc);
    orc_dequant(acc, gamma, s, M, N, residual, y, NULL);
    if (acc_out) memcpy(acc_out, acc, sizeof(int32_t) * (size_t)(M * N));
    if (xq_out) memcpy(xq_out, xq, (size_t)(M * K));
    if (s_out) memcpy(s_out, s, sizeof(float) * (size_t)M);
    if (xsum_out) memcpy(xsum_out, xsum, sizeof(int32_t) * (size_t)M);
    free(xf); free(xq); free(s); free(xsum); free(acc);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* subln RMSNorm with unit weight over one token's f features ([news] BitLinear
 * list: sub-layer normalisation; [card] "Method Adaptation": subln).
 * Returns r = 1 / sqrtf(float(sum h^2 / f) + eps); hn = h * r.              */
float orc_subln_rms(const float* h, int64_t f, float* hn) {
    double ss = 0.0;
    for (int64_t j = 0; j < f; ++j) ss += (double)h[j] * (double)h[j];
    float ms = (float)(ss / (double)f);
    float r = 1.0f / sqrtf(ms + ORC_RMS_EPS);
    for (int64_t j = 0; j < f; ++j) hn[j] = h[j] * r;
    return r;
}

/* ReLU^2 gating of one element ([news]: ReLU^2 in the FFN sub-layer; [card]
 * "Method Adaptation": ReLU^2 feed-forward): (max(g, 0))^2 * u, each product
 * rounded to fp32.                                                          */
float orc_relu2_gate(float g, float u) {
    float t = g > 0.0f ? g : 0.0f;
    return (t * t) * u;
}

/* One FFN sub-layer on M tokens: d -> f (gate, up) -> f -> d (down).
 *   xq, s = quant(x); g = deq(Wg . xq); u = deq(Wu . xq); h = relu(g)^2 * u;
 *   hn = subln(h); q2, s2 = quant(hn); y = bf16(residual + deq(Wd . q2)).
 * Packed weights: Wg, Wu [f, d/4]; Wd [d, f/4]. x, residual, y: [M, d] bf16.
 * Optional outputs (NULL to skip): h_out [M, f] fp32, q2_out [M, f] int8,
 * s2_out [M], r_out [M], accd_out [M, d].                                    */
int orc_ffn_layer(const uint8_t* Wg, float gg, const uint8_t* Wu, float gu,
                  const uint8_t* Wd, float gd, int64_t d, int64_t f,
                  const uint16_t* x, int64_t M, const uint16_t* residual, uint16_t* y,
                  float* h_out, int8_t* q2_out, float* s2_out, float* r_out, int32_t* accd_out) {
    float* xf = (float*)malloc(sizeof(float) * (size_t)(M * d));
    int8_t* xq = (int8_t*)malloc((size_t)(M * d));
    float* s = (float*)malloc(sizeof(float) * (size_t)M);
    int32_t* accg = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * f));
    int32_t* accu = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * f));
    float* h = (float*)malloc(sizeof(float) * (size_t)(M * f));
    float* hn = (float*)malloc(sizeof(float) * (size_t)(M * f));
    int8_t* q2 = (int8_t*)malloc((size_t)(M * f));
    float* s2 = (float*)malloc(sizeof(float) * (size_t)M);
    int32_t* accd = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * d));
    int rc = 0;
    if (!xf || !xq || !s || !accg || !accu || !h || !hn || !q2 || !s2 || !accd) {
        rc = -1;
        goto done;
    }
    orc_bf16_to_f32_array(x, M * d, xf);
    orc_quant_act(xf, M, d, xq, s, NULL);
    orc_int_gemm_packed(Wg, xq, M, f, d, accg);
    orc_int_gemm_packed(Wu, xq, M, f, d, accu);
    for (int64_t m = 0; m < M; ++m) {
        float deqg = gg / s[m];
        float dequ = gu / s[m];
        for (int64_t j = 0; j < f; ++j) {
            float g = (float)accg[m * f + j] * deqg;
            float u = (float)accu[m * f + j] * dequ;
            h[m * f + j] = orc_relu2_gate(g, u);
        }
        float r = orc_subln_rms(h + m * f, f, hn + m * f);
        if (r_out) r_out[m] = r;
    }
    orc_quant_act(hn, M, f, q2, s2, NULL);
    orc_int_gemm_packed(Wd, q2, M, d, f, accd);
    orc_dequant(accd, gd, s2, M, d, residual, y, NULL);
    if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)(M * f));
    if (q2_out) memcpy(q2_out, q2, (size_t)(M * f));
    if (s2_out) memcpy(s2_out, s2, sizeof(float) * (size_t)M);
    if (accd_out) memcpy(accd_out, accd, sizeof(int32_t) * (size_t)(M * d));
done:
    free(xf); free(xq); free(s); free(accg); free(accu); free(h); free(hn); free(q2); free(s2); free(accd);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Several BitLinear projections of one input: the weight matrices are stacked
 * row-wise (for example the attention's query, key and value projections, which
 * read the same x), each keeps its own absmean gamma ([card] "Method
 * Adaptation": absmean per weight tensor), and the input may first pass through
 * a unit-weight RMSNorm (the block's pre-norm, and the subln in front of the
 * attention output projection; [news] BitLinear list, [card] "Method
 * Adaptation": subln). Reading: the same RMSNorm as the FFN's subln (sum of
 * squares in fp64, r = 1 / sqrtf(float(sum / K) + 1e-5f), xn = x * r in fp32,
 * not rounded to bf16 before the quantisation).
 *   Wp [N, K/4], N = sum of seg_rows[0..nseg-1]; rows of segment i use gammas[i].
 *   x, residual, y: [M, K], [M, N], [M, N] bf16 bits; acc_out [M, N] or NULL.   */
int orc_forward_ex(const uint8_t* Wp, const float* gammas, const int64_t* seg_rows, int64_t nseg,
                   int64_t K, const uint16_t* x, int64_t M, int64_t rmsnorm,
                   const uint16_t* residual, uint16_t* y, int32_t* acc_out) {
    int64_t N = 0;
    for (int64_t i = 0; i < nseg; ++i) N += seg_rows[i];
    float* xf = (float*)malloc(sizeof(float) * (size_t)(M * K));
    float* xn = (float*)malloc(sizeof(float) * (size_t)(M * K));
    int8_t* xq = (int8_t*)malloc((size_t)(M * K));
    float* s = (float*)malloc(sizeof(float) * (size_t)M);
    int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * N));
    int rc = 0;
    if (!xf || !xn || !xq || !s || !acc) {
        rc = -1;
        goto done;
    }
    orc_bf16_to_f32_array(x, M * K, xf);
    for (int64_t m = 0; m < M; ++m) {
        if (rmsnorm)
            orc_subln_rms(xf + m * K, K, xn + m * K);
        else
            memcpy(xn + m * K, xf + m * K, sizeof(float) * (size_t)K);
    }
    orc_quant_act(xn, M, K, xq, s, NULL);
    orc_int_gemm_packed(Wp, xq, M, N, K, acc);
    for (int64_t m = 0; m < M; ++m) {
        int64_t n = 0;
        for (int64_t i = 0; i < nseg; ++i) {
            float deq = gammas[i] / s[m];
            for (int64_t e = 0; e < seg_rows[i]; ++e, ++n) {
                float v = (float)acc[m * N + n] * deq;
                if (residual) v = orc_bf16_to_f32(residual[m * N + n]) + v;
                y[m * N + n] = orc_f32_to_bf16(v);
            }
        }
    }
    if (acc_out) memcpy(acc_out, acc, sizeof(int32_t) * (size_t)(M * N));
done:
    free(xf); free(xn); free(xq); free(s); free(acc);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Per-row absmean variant of the weight path (one gamma per output row instead
 * of one per tensor; [card] "Method Adaptation" gives one absmean per weight
 * tensor, so this is a variant of that reading): gamma_n = mean_k |W[n,k]|
 * (fp64 sum in k order, fp64 division by K, one rounding to fp32), row n
 * ternarised with its own gamma_n, then packed as usual.                      */
int orc_pack_weights_rowwise(const float* W, int64_t N, int64_t K, uint8_t* Wp, float* gammas) {
    int8_t* q = (int8_t*)malloc((size_t)(N * K));
    if (!q) return -1;
    for (int64_t n = 0; n < N; ++n) {
        gammas[n] = orc_absmean(W + n * K, K);
        orc_ternarize(W + n * K, K, gammas[n], q + n * K);
    }
    orc_pack(q, N, K, Wp);
    free(q);
    return 0;
}

/* Forward with per-row gammas: y[m, n] = bf16([res +] float(acc) * (gamma_n / s_m)). */
int orc_forward_rowwise(const uint8_t* Wp, const float* gammas, int64_t N, int64_t K,
                        const uint16_t* x, int64_t M, const uint16_t* residual,
                        uint16_t* y, int32_t* acc_out) {
    float* xf = (float*)malloc(sizeof(float) * (size_t)(M * K));
    int8_t* xq = (int8_t*)malloc((size_t)(M * K));
    float* s = (float*)malloc(sizeof(float) * (size_t)M);
    int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * N));
    int rc = 0;
    if (!xf || !xq || !s || !acc) {
        rc = -1;
        goto done;
    }
    orc_bf16_to_f32_array(x, M * K, xf);
    orc_quant_act(xf, M, K, xq, s, NULL);
    orc_int_gemm_packed(Wp, xq, M, N, K, acc);
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            float deq = gammas[n] / s[m];
            float v = (float)acc[m * N + n] * deq;
            if (residual) v = orc_bf16_to_f32(residual[m * N + n]) + v;
            y[m * N + n] = orc_f32_to_bf16(v);
        }
    }
    if (acc_out) memcpy(acc_out, acc, sizeof(int32_t) * (size_t)(M * N));
done:
    free(xf); free(xq); free(s); free(acc);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Tensor-parallel pieces of the weight path and of the FFN sub-layer. The pages
 * give no distributed detail (paper card, "Limits"); this is the library's
 * split of the same computation over P ranks: rank r owns rows [c0, c1) of the
 * gate and up weights and the same columns of the down weight. Composed over
 * the ranks (sums and maxima exchanged between them), the pieces give exactly
 * orc_pack_weights and orc_ffn_layer on the whole tensors.                   */

/* fp64 sum of |W| over one shard (row-major order), the term each rank adds to
 * the per-tensor absmean of [card] "Method Adaptation".                       */
double orc_absmean_sum(const float* W, int64_t n) {
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += fabs((double)W[i]);
    return s;
}

/* Ternarise and pack one shard with the gamma of the whole tensor:
 * gamma = fp32(total_sum / total_count), the fp64 sum and count over all shards. */
int orc_pack_weights_global(const float* W, int64_t N, int64_t K, double total_sum, int64_t total_count,
                            uint8_t* Wp, float* gamma_out) {
    int8_t* q = (int8_t*)malloc((size_t)(N * K));
    if (!q) return -1;
    float gamma = (float)(total_sum / (double)total_count);
    orc_ternarize(W, N * K, gamma, q);
    orc_pack(q, N, K, Wp);
    free(q);
    *gamma_out = gamma;
    return 0;
}

/* Rank-local first half of the FFN: x is quantised whole (every rank holds it),
 * the rank's fl gate and up rows give h = relu(g)^2 * u as in orc_ffn_layer, and
 * per token the rank's share of the subln statistics: ss = sum_j h_j^2 (fp64,
 * j in order) and hmax = max_j |h_j| over its fl columns.                      */
int orc_ffn_tp_up(const uint8_t* Wg, float gg, const uint8_t* Wu, float gu, int64_t d, int64_t fl,
                  const uint16_t* x, int64_t M, float* h, double* ss, float* hmax) {
    float* xf = (float*)malloc(sizeof(float) * (size_t)(M * d));
    int8_t* xq = (int8_t*)malloc((size_t)(M * d));
    float* s = (float*)malloc(sizeof(float) * (size_t)M);
    int32_t* accg = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * fl));
    int32_t* accu = (int32_t*)malloc(sizeof(int32_t) * (size_t)(M * fl));
    int rc = 0;
    if (!xf || !xq || !s || !accg || !accu) {
        rc = -1;
        goto done;
    }
    orc_bf16_to_f32_array(x, M * d, xf);
    orc_quant_act(xf, M, d, xq, s, NULL);
    orc_int_gemm_packed(Wg, xq, M, fl, d, accg);
    orc_int_gemm_packed(Wu, xq, M, fl, d, accu);
    for (int64_t m = 0; m < M; ++m) {
        float deqg = gg / s[m];
        float dequ = gu / s[m];
        double acc_ss = 0.0;
        float mx = 0.0f;
        for (int64_t j = 0; j < fl; ++j) {
            float g = (float)accg[m * fl + j] * deqg;
            float u = (float)accu[m * fl + j] * dequ;
            float hv = orc_relu2_gate(g, u);
            h[m * fl + j] = hv;
            acc_ss += (double)hv * (double)hv;
            if (fabsf(hv) > mx) mx = fabsf(hv);
        }
        ss[m] = acc_ss;
        hmax[m] = mx;
    }
done:
    free(xf); free(xq); free(s); free(accg); free(accu);
    return rc;
}

/* Rank-local second half: with the statistics of all ranks (ss_all: the sum of
 * the ranks' ss; hmax_all: their maximum) the subln factor and the
 * requantisation scale are those of the whole h:
 *   r  = 1 / sqrtf(float(ss_all / f_total) + eps)      (orc_subln_rms)
 *   s2 = 127 / max(max_j |fl(h_j r)|, 1e-5) = 127 / max(fl(hmax_all r), 1e-5)
 * (rounding is monotonic and r > 0, so the largest |fl(h_j r)| is fl(max|h_j| r));
 * the rank quantises its columns fl(h_j r) with s2 and contracts them with its
 * down columns: acc[m, n] = sum_{j in the rank's columns} Wd[n, j] q2[m, j].   */
int orc_ffn_tp_down(const uint8_t* Wd, int64_t d, int64_t fl, int64_t f_total, const float* h, int64_t M,
                    const double* ss_all, const float* hmax_all, int32_t* acc, float* s2) {
    int8_t* q2 = (int8_t*)malloc((size_t)(M * fl));
    if (!q2) return -1;
    for (int64_t m = 0; m < M; ++m) {
        float ms = (float)(ss_all[m] / (double)f_total);
        float r = 1.0f / sqrtf(ms + ORC_RMS_EPS);
        float sm = ORC_QB / fmaxf(hmax_all[m] * r, ORC_X_EPS);
        for (int64_t j = 0; j < fl; ++j) {
            float v = rintf((h[m * fl + j] * r) * sm);
            if (v > 127.0f) v = 127.0f;
            if (v < -128.0f) v = -128.0f;
            q2[m * fl + j] = (int8_t)v;
        }
        s2[m] = sm;
    }
    orc_int_gemm_packed(Wd, q2, M, d, fl, acc);
    free(q2);
    return 0;
}
