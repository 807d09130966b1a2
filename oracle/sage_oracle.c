/*
 * sage_oracle.c -- plain, slow, scalar CPU oracle for the SageAttention
 * quantized attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library) shares no code, header, table or constant generator with it.
 *
 * Sources (cited by page title and section):
 *   [SA2]  "SageAttention2: Efficient Attention with Thorough Outlier Smoothing
 *          and Per-thread INT4 Quantization" -- reading note at
 *          zhaifeiyue.github.io/papers/2411.10958/detail, "Algorithm 1:
 *          SageAttention2" and its line-by-line commentary, "5. Numerical
 *          Considerations".
 *   [SA1]  SageAttention note at zhaifeiyue.github.io/papers/2410.02367
 *          (Smooth K: gamma(K) = K - mean(K), exact by softmax shift invariance).
 *   [SA3]  SageAttention3 note at zhaifeiyue.github.io/papers/2505.11594
 *          (two-level P quantisation: per-token FP32 s_P1 with 448*6 = 2688,
 *          per-block E4M3 s_P2; NVFP4 = E2M1 values + E4M3 scale per 16).
 *   [BLOG] "SageAttention量化加速框架" (blog.gitcode.com), section
 *          "数学公式：分层量化的数值稳定性保障": X_int8 = round(X / S).
 *   [FAvsSA] "FlashAttention vs SageAttention" (kenforever1.github.io source
 *          analysis), sections "Online Softmax" (m, l, rescale update) and
 *          "精度与量化策略" (per-block INT8, per-channel FP8 V, smooth_k).
 *
 * Readings taken where the pages are silent:
 *   - means are summed in fp64 and rounded once to fp32;
 *   - INT8 scale = amax / 127 (fp32 division), code = clamp(rint(x / scale)),
 *     x / scale an IEEE fp32 division, rint = round-half-to-even;
 *   - E4M3 is the OCP "fn" variant (bias 7, max 448, no infinities), encoded
 *     with round-to-nearest-even and saturation to +-448;
 *   - E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}, round-to-nearest-even, saturate
 *     to +-6;
 *   - sm_scale multiplies the dequantised score (after + delta_S);
 *   - the online softmax is blocked over `tile` keys (the kernel's K tile);
 *     l is summed over the fp32 P~ before P is quantised.
 */
#include "sage_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 ("fn"): 1 sign, 4 exponent (bias 7), 3 mantissa bits.            */
/* Normal:    (8 + m) * 2^(e - 10)   for e in 1..15 (e=15,m=7 is NaN)         */
/* Subnormal:  m * 2^-9              for e = 0                               */
/* ------------------------------------------------------------------------ */
float or_e4m3_decode(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    float v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexpf((float)m, -9);
    else        v = ldexpf((float)(8 + m), e - 10);
    return s ? -v : v;
}

uint8_t or_e4m3_encode(float x)
{
    uint8_t sign;
    float a, quantum, q, val;
    int ex, e, m;
    if (isnan(x)) return 0x7F;
    sign = signbit(x) ? 0x80 : 0x00;
    a = fabsf(x);
    if (a >= 448.0f) return sign | 0x7E;               /* saturate to 448 */
    if (a < ldexpf(1.0f, -6)) {
        quantum = ldexpf(1.0f, -9);                     /* subnormal spacing */
    } else {
        frexpf(a, &ex);                                 /* a = f * 2^ex, f in [0.5,1) */
        quantum = ldexpf(1.0f, (ex - 1) - 3);           /* 3 mantissa bits */
    }
    q = rintf(a / quantum);                             /* exact scaling, RNE */
    val = q * quantum;
    if (val == 0.0f) return sign;
    if (val < ldexpf(1.0f, -6)) {
        m = (int)(val / ldexpf(1.0f, -9));
        return sign | (uint8_t)m;
    }
    frexpf(val, &ex);
    e = (ex - 1) + 7;
    m = (int)(val / ldexpf(1.0f, ex - 1) * 8.0f) - 8;
    return sign | (uint8_t)(e << 3) | (uint8_t)m;
}

/* ------------------------------------------------------------------------ */
/* FP4 E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit.                    */
/* Normal: (2 + m) * 2^(e - 2) for e in 1..3;  subnormal: m * 0.5 for e = 0  */
/* ------------------------------------------------------------------------ */
float or_e2m1_decode(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    float v = (e == 0) ? 0.5f * (float)m : ldexpf((float)(2 + m), e - 2);
    return s ? -v : v;
}

uint8_t or_e2m1_encode(float x)
{
    uint8_t sign;
    float a, quantum, q, val;
    int ex, e, m;
    if (isnan(x)) return 0x7;                            /* no NaN in E2M1: saturate */
    sign = signbit(x) ? 0x8 : 0x0;
    a = fabsf(x);
    if (a >= 6.0f) return sign | 0x7;
    if (a < 1.0f) {
        quantum = 0.5f;
    } else {
        frexpf(a, &ex);
        quantum = ldexpf(1.0f, (ex - 1) - 1);            /* 1 mantissa bit */
    }
    q = rintf(a / quantum);
    val = q * quantum;
    if (val == 0.0f) return sign;
    if (val < 1.0f) return sign | 0x1;                   /* 0.5 */
    frexpf(val, &ex);
    e = (ex - 1) + 1;
    m = (int)(val / ldexpf(1.0f, ex - 1) * 2.0f) - 2;
    return sign | (uint8_t)(e << 1) | (uint8_t)m;
}

/* ------------------------------------------------------------------------ */
/* Smoothing statistics.                                                     */
/* ------------------------------------------------------------------------ */

/* mean over rows of X[rows, d]  ([SA1] Smooth K; [SA2] Alg. 1 "K = K - mean(K)",
 * "q_i = mean(Q_i)").  fp64 sum, one rounding to fp32. */
int or_mean_rows(const float *X, int64_t rows, int d, float *mean)
{
    int64_t n;
    int c;
    if (rows <= 0 || d <= 0) return -1;
    for (c = 0; c < d; ++c) {
        double acc = 0.0;
        for (n = 0; n < rows; ++n) acc += (double)X[n * d + c];
        mean[c] = (float)(acc / (double)rows);
    }
    return 0;
}

/* Per-block row means: block i covers rows [i*blk, min((i+1)*blk, rows)). */
int or_block_means(const float *X, int64_t rows, int d, int blk, float *means)
{
    int64_t T = (rows + blk - 1) / blk, i;
    for (i = 0; i < T; ++i) {
        int64_t r0 = i * blk, r1 = r0 + blk < rows ? r0 + blk : rows;
        if (or_mean_rows(X + r0 * d, r1 - r0, d, means + i * d)) return -1;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Per-block symmetric INT8 quantisation ([BLOG] X_int8 = round(X / S);       */
/* [SA2] Alg. 1 psi_Q(Q_i - q_i), psi_K(K_j); [FAvsSA] per_block INT8).      */
/* x = X - mean (fp32 subtraction; mean is [d] for all rows, or [T, d] one   */
/* per block), scale = amax_block |x| / 127, code = clamp(rint(x / scale)).  */
/* ------------------------------------------------------------------------ */
int or_quant_int8(const float *X, int64_t rows, int d, int blk,
                  const float *mean, int mean_per_block,
                  int8_t *out, float *scale)
{
    int64_t T = (rows + blk - 1) / blk, i, n;
    int c;
    if (rows <= 0 || d <= 0 || blk <= 0) return -1;
    for (i = 0; i < T; ++i) {
        int64_t r0 = i * blk, r1 = r0 + blk < rows ? r0 + blk : rows;
        const float *mu = mean ? (mean_per_block ? mean + i * d : mean) : NULL;
        float amax = 0.0f, s;
        for (n = r0; n < r1; ++n)
            for (c = 0; c < d; ++c) {
                float x = mu ? X[n * d + c] - mu[c] : X[n * d + c];
                float ax = fabsf(x);
                if (ax > amax) amax = ax;
            }
        s = amax / 127.0f;
        scale[i] = s;
        for (n = r0; n < r1; ++n)
            for (c = 0; c < d; ++c) {
                float x = mu ? X[n * d + c] - mu[c] : X[n * d + c];
                float q;
                if (s == 0.0f) { out[n * d + c] = 0; continue; }
                q = rintf(x / s);
                if (q > 127.0f) q = 127.0f;
                if (q < -127.0f) q = -127.0f;
                out[n * d + c] = (int8_t)q;
            }
    }
    return 0;
}

/* Per-channel FP8 E4M3 quantisation of V ([SA2] Alg. 1 (delta_V, V^) = psi_V(V);
 * "Deep Analysis" 3: V -> FP8 E4M3 per-channel):
 * scale_v[c] = amax_n |V[n, c]| / 448, code = E4M3(V / scale_v[c]). */
int or_quant_fp8_per_channel(const float *V, int64_t rows, int d, uint8_t *out, float *scale_v)
{
    int64_t n;
    int c;
    if (rows <= 0 || d <= 0) return -1;
    for (c = 0; c < d; ++c) {
        float amax = 0.0f, s;
        for (n = 0; n < rows; ++n) {
            float ax = fabsf(V[n * d + c]);
            if (ax > amax) amax = ax;
        }
        s = amax / 448.0f;
        scale_v[c] = s;
        for (n = 0; n < rows; ++n)
            out[n * d + c] = (s == 0.0f) ? 0 : or_e4m3_encode(V[n * d + c] / s);
    }
    return 0;
}

/* delta_S[i, j] = q_i . gamma(K_j) with gamma(K) = K - mean(K) (fp32), summed in
 * fp64 ([SA2] Alg. 1 "GEMV(q_i, K_j^T)"; commentary: the row-constant term
 * b = q_i.k^T + gamma(Q_i).k^T is dropped). qbar [Tm, d], K [N, d] -> dS [Tm, N]. */
int or_delta_s(const float *qbar, int64_t Tm, const float *K, const float *km,
               int64_t N, int d, float *dS)
{
    int64_t i, j;
    int c;
    float *g = (float *)malloc(sizeof(float) * (size_t)d);
    if (!g) return -2;
    for (j = 0; j < N; ++j) {
        for (c = 0; c < d; ++c) g[c] = km ? K[j * d + c] - km[c] : K[j * d + c];
        for (i = 0; i < Tm; ++i) {
            double acc = 0.0;
            for (c = 0; c < d; ++c) acc += (double)qbar[i * d + c] * (double)g[c];
            dS[i * N + j] = (float)acc;
        }
    }
    free(g);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 quantisation ([SA3]: E2M1 values, one E4M3 scale per 16 elements;  */
/* block scale = E4M3(amax16 / 6), value = E2M1(x / decode(block scale))).  */
/* ------------------------------------------------------------------------ */

/* groups of 16 along d (Q, K): codes [rows, d] (one code per byte), sf [rows, d/16] */
int or_quant_nvfp4_rows(const float *X, int64_t rows, int d, int blk,
                        const float *mean, int mean_per_block,
                        uint8_t *codes, uint8_t *sf)
{
    int64_t n;
    int g, c;
    if (rows <= 0 || d <= 0 || d % 16) return -1;
    for (n = 0; n < rows; ++n) {
        const float *mu = mean ? (mean_per_block ? mean + (n / blk) * d : mean) : NULL;
        for (g = 0; g < d / 16; ++g) {
            float x[16], amax = 0.0f, sd;
            uint8_t s8;
            for (c = 0; c < 16; ++c) {
                int cc = g * 16 + c;
                x[c] = mu ? X[n * d + cc] - mu[cc] : X[n * d + cc];
                if (fabsf(x[c]) > amax) amax = fabsf(x[c]);
            }
            s8 = or_e4m3_encode(amax / 6.0f);
            sf[n * (d / 16) + g] = s8;
            sd = or_e4m3_decode(s8);
            for (c = 0; c < 16; ++c)
                codes[n * d + g * 16 + c] = (sd == 0.0f) ? 0 : or_e2m1_encode(x[c] / sd);
        }
    }
    return 0;
}

/* groups of 16 consecutive tokens per channel (V, the reduction axis of P V):
 * codes [rows, d], sf [ceil(rows/16), d]; a partial last group uses its valid rows. */
int or_quant_nvfp4_cols(const float *V, int64_t rows, int d, uint8_t *codes, uint8_t *sf)
{
    int64_t G = (rows + 15) / 16, g, n;
    int c;
    if (rows <= 0 || d <= 0) return -1;
    for (g = 0; g < G; ++g) {
        int64_t r0 = g * 16, r1 = r0 + 16 < rows ? r0 + 16 : rows;
        for (c = 0; c < d; ++c) {
            float amax = 0.0f, sd;
            uint8_t s8;
            for (n = r0; n < r1; ++n)
                if (fabsf(V[n * d + c]) > amax) amax = fabsf(V[n * d + c]);
            s8 = or_e4m3_encode(amax / 6.0f);
            sf[g * d + c] = s8;
            sd = or_e4m3_decode(s8);
            for (n = r0; n < r1; ++n)
                codes[n * d + c] = (sd == 0.0f) ? 0 : or_e2m1_encode(V[n * d + c] / sd);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Blocked online-softmax attention ([SA2] Alg. 1 inner loop; [FAvsSA]       */
/* "Online Softmax").  One row at a time, keys in tiles of `tile`:           */
/*   S      = dot(Qv[r], Kv[c]) * row_scale[r] * col_scale[c] (+ dS) * sm    */
/*   m_new  = max(m, rowmax(S))                                              */
/*   P~     = exp(S - m_new)                                                 */
/*   l      = exp(m - m_new) * l + rowsum(P~)                                */
/*   O_t    = quant(P~) @ V_tile        (level 1: fresh per tile)            */
/*   O      = exp(m - m_new) * O + O_t  (level 2: FP32 buffer)               */
/*   out    = O / l  (/ 448 * scale_v for the E4M3 P path)                   */
/* p_mode 0: P unquantised (identity codec)                                  */
/* p_mode 1: P^ = E4M3(P~ * 448), final / 448 * out_scale ([SA2] static scale)*/
/* p_mode 2: SA3 two-level: s_P1 = rowmax_tile(P~) / 2688 (fp32, per row per */
/*           tile); P2 = P~ / s_P1; s_P2 = E4M3(amax16(P2) / 6) per 16 keys; */
/*           P^ = E2M1(P2 / s_P2); O_t = s_P1 * sum(P^ s_P2 V)                */
/* round32: every state/score operation rounded to fp32 (the kernel's        */
/* precision); 0 keeps everything in fp64 (used by the fp64 pins).           */
/* ------------------------------------------------------------------------ */
#define RND(x) (round32 ? (double)(float)(x) : (double)(x))

int or_attn_core(const double *Qv, const double *Kv, const double *Vv,
                 const double *row_scale, const double *col_scale,
                 const float *dS, int bq, const double *out_scale,
                 int64_t N, int d, int tile, int causal, double sm_scale,
                 int p_mode, int round32,
                 int64_t r0, int64_t r1, double *out, double *lse)
{
    int64_t r, j0, c;
    int k;
    double *S = (double *)malloc(sizeof(double) * (size_t)tile);
    double *P = (double *)malloc(sizeof(double) * (size_t)tile);
    double *O = (double *)malloc(sizeof(double) * (size_t)d);
    double *Ot = (double *)malloc(sizeof(double) * (size_t)d);
    if (!S || !P || !O || !Ot) { free(S); free(P); free(O); free(Ot); return -2; }
    if (r0 < 0 || r1 > N || tile <= 0 || (p_mode == 2 && tile % 16)) {
        free(S); free(P); free(O); free(Ot);
        return -1;
    }
    for (r = r0; r < r1; ++r) {
        double m = -INFINITY, l = 0.0;
        for (k = 0; k < d; ++k) O[k] = 0.0;
        for (j0 = 0; j0 < N; j0 += tile) {
            int64_t j1 = j0 + tile < N ? j0 + tile : N;
            int64_t n;
            double rowmax = -INFINITY, m_new, alpha, rowsum = 0.0, pscale = 1.0;
            if (causal && j1 > r + 1) j1 = r + 1;
            if (j1 <= j0) break;
            n = j1 - j0;
            /* scores: S = psi^-1(Q^ K^T) + GEMV(q_i, K^T), times sm_scale */
            for (c = 0; c < n; ++c) {
                double dot = 0.0, s;
                for (k = 0; k < d; ++k) dot += Qv[r * d + k] * Kv[(j0 + c) * d + k];
                s = RND(dot);
                if (row_scale) s = RND(s * row_scale[r]);
                if (col_scale) s = RND(s * col_scale[j0 + c]);
                if (dS) s = RND(s + (double)dS[(r / bq) * N + (j0 + c)]);
                s = RND(s * sm_scale);
                S[c] = s;
                if (s > rowmax) rowmax = s;
            }
            m_new = m > rowmax ? m : rowmax;
            alpha = (m == -INFINITY) ? 0.0 : RND(exp(m - m_new));
            for (c = 0; c < n; ++c) {
                P[c] = RND(exp(S[c] - m_new));
                rowsum = RND(rowsum + P[c]);
            }
            l = RND(RND(alpha * l) + rowsum);
            /* quantise P~ */
            if (p_mode == 1) {
                for (c = 0; c < n; ++c)
                    P[c] = (double)or_e4m3_decode(or_e4m3_encode((float)RND(P[c] * 448.0)));
            } else if (p_mode == 2) {
                double pmax = 0.0, sP1;
                for (c = 0; c < n; ++c) if (P[c] > pmax) pmax = P[c];
                sP1 = RND(pmax / 2688.0);
                pscale = sP1;
                for (c = 0; c < n; c += 16) {
                    int64_t g1 = c + 16 < n ? c + 16 : n, cc;
                    double amax = 0.0, sd;
                    uint8_t s8;
                    if (sP1 == 0.0) { for (cc = c; cc < g1; ++cc) P[cc] = 0.0; continue; }
                    for (cc = c; cc < g1; ++cc) {
                        P[cc] = RND(P[cc] / sP1);
                        if (P[cc] > amax) amax = P[cc];
                    }
                    s8 = or_e4m3_encode((float)RND(amax / 6.0));
                    sd = (double)or_e4m3_decode(s8);
                    for (cc = c; cc < g1; ++cc)
                        P[cc] = (sd == 0.0) ? 0.0
                                : (double)or_e2m1_decode(or_e2m1_encode((float)RND(P[cc] / sd))) * sd;
                }
            }
            /* level 1: O_t = P^ V_j (fresh accumulator) */
            for (k = 0; k < d; ++k) {
                double acc = 0.0;
                for (c = 0; c < n; ++c) acc += P[c] * Vv[(j0 + c) * d + k];
                Ot[k] = RND(acc);
                if (p_mode == 2) Ot[k] = RND(Ot[k] * pscale);
            }
            /* level 2: O = diag(exp(m - m_new)) O + O_t */
            for (k = 0; k < d; ++k) O[k] = RND(RND(alpha * O[k]) + Ot[k]);
            m = m_new;
        }
        for (k = 0; k < d; ++k) {
            double o = RND(O[k] / l);
            if (p_mode == 1) o = RND(o / 448.0);
            if (out_scale) o = RND(o * out_scale[k]);
            out[(r - r0) * d + k] = o;
        }
        /* log-sum-exp of the row's scores S (natural log): m + ln l, where l
           is the running sum of exp(S - m) over the visible keys */
        if (lse) lse[r - r0] = (l > 0.0) ? m + log(l) : -INFINITY;
    }
    free(S); free(P); free(O); free(Ot);
    return 0;
}

/* Textbook attention in fp64: out = softmax(Q K^T * sm_scale) V (two passes). */
int or_attn_naive_f64(const double *Q, const double *K, const double *V,
                      int64_t N, int d, int causal, double sm_scale,
                      int64_t r0, int64_t r1, double *out)
{
    int64_t r, c;
    int k;
    double *S = (double *)malloc(sizeof(double) * (size_t)N);
    if (!S) return -2;
    if (r0 < 0 || r1 > N) { free(S); return -1; }
    for (r = r0; r < r1; ++r) {
        int64_t n = causal ? r + 1 : N;
        double mx = -INFINITY, sum = 0.0;
        for (c = 0; c < n; ++c) {
            double dot = 0.0;
            for (k = 0; k < d; ++k) dot += Q[r * d + k] * K[c * d + k];
            S[c] = dot * sm_scale;
            if (S[c] > mx) mx = S[c];
        }
        for (c = 0; c < n; ++c) { S[c] = exp(S[c] - mx); sum += S[c]; }
        for (k = 0; k < d; ++k) {
            double acc = 0.0;
            for (c = 0; c < n; ++c) acc += S[c] * V[c * d + k];
            out[(r - r0) * d + k] = acc / sum;
        }
    }
    free(S);
    return 0;
}
