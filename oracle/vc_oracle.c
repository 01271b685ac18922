/*
 * vc_oracle.c -- plain, slow CPU reference for VC-Attention (V-Smooth prep +
 * ExpCast-FP8 attention forward).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check,
 * and the benchmark's CPU-baseline leg and reference arm may load this library.  The CUDA path never
 * calls it, and it shares no code, header, table or constant with the CUDA
 * path: every format and formula here is written from its definition.
 *
 * Sources (the method is described only in prose on these pages):
 *   [ChooseAI/V-Smooth]  chooseai.io news 7051, section
 *                        "核心方法之一：V-Smooth 把 value 的离群值收拢"
 *   [ChooseAI/ExpCast]   chooseai.io news 7051, section
 *                        "核心方法之二：ExpCast-FP8 换掉 softmax 里的指数"
 *   [Clarity]            theclarity.today, "Quantizing value residuals and
 *                        casting softmax to FP8 speeds Nunchux's attention
 *                        kernel 1.46x on an H200" (V-Smooth and ExpCast paragraphs)
 *   [MarkTechPost]       zerohour.day summary "Nunchux AI Introduces
 *                        VC-Attention ...", key-facts bullets
 *   [RuntimeWire]        "Nunchux speeds video diffusion with value smoothing
 *                        and FP8 softmax casting", section "The arithmetic
 *                        behind the speedup"
 *
 * Readings where the pages are silent (the CUDA path takes the same ones):
 *   - E4M3 is the OCP FP8 E4M3 ("fn") format: bias 7, no infinities, 0x7F NaN,
 *     max 448, subnormals m * 2^-9.  Encoding rounds to nearest, ties to even,
 *     and saturates to +-448.
 *   - k-means: strided init c_k = v[floor(k*n/C)]; `iters` assignment passes
 *     with iters-1 centroid updates in between; ties go to the lowest index; an
 *     empty cluster keeps its centroid.  Distances in fp64.
 *   - Regroup: stable counting sort of token indices by cluster id; blocks are
 *     consecutive runs of `bk` tokens in that order (a block may straddle
 *     clusters); the last block holds only the valid rows.
 *   - K: one amax scale per block (sk = amax/448); Q: one scale per token.
 *   - V: block mean mu_b (fp64 mean rounded to fp32), residual r = v - mu_b in
 *     fp32, one residual scale per channel per head (s_c = amax_c/448).
 *   - ExpCast: per row an integer reference M = ceil(max_j A*s_j / 8) kept
 *     online over the tiles; byte = max(0, rne(A*s_j + 56 + beta - 8M)) with
 *     beta an integer, a single rounding of the exact value.
 *   - Mean restore: O += l_b * mu_b per tile with l_b = sum of the decoded
 *     bytes of the tile, all terms rescaled by 2^-k when M rises by k.
 *   - NVFP4 (the 4-bit residual [MarkTechPost]: the V residual is quantised
 *     per channel to E4M3 or to NVFP4): E2M1 values (OCP MX FP4: sign, 2
 *     exponent bits with bias 1, 1 mantissa bit; max 6) in blocks of 16 along
 *     the reduction axis, each block with a UE4M3 scale s = E4M3(amax/6); a
 *     value x is coded
 *     E2M1(x * (1/s)), with 1/s and the product rounded to fp32, E2M1 rounding
 *     to nearest (ties to the even code) and saturating at 6; a zero scale
 *     codes zeros.  The V residual keeps one fp32 scale per channel,
 *     s_c = amax_c/(6*448), before its 16-token blocks.  The PV product of the
 *     4-bit path takes P in the same 16-key blocks, re-coded from the ExpCast
 *     byte's E4M3 value.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define VO_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* bf16 input: the upper 16 bits of an IEEE binary32.                        */
/* ------------------------------------------------------------------------ */
static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------ */
/* E4M3 codec, from the format definition.                                   */
/* ------------------------------------------------------------------------ */

/* Value of an E4M3 byte: sign bit 7, exponent bits 6..3 (bias 7), mantissa
 * bits 2..0.  Exponent field 0 is subnormal (m/8 * 2^-6); 0x7F/0xFF are NaN. */
VO_API double vo_e4m3_value(uint8_t code) {
    int sign = code >> 7;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Round a float to the nearest E4M3 value, ties to the even code, saturating
 * to +-448.  The nearest code is found by bisection over the 127 non-negative
 * finite codes, whose values increase with the code. */
VO_API uint8_t vo_e4m3_encode(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (isnan(x)) return 0x7F;
    if (a >= 448.0) return sign | 0x7E;
    int lo = 0, hi = 126; /* value(lo) <= a < value(hi) after the loop */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (vo_e4m3_value((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid;
    }
    double dlo = a - vo_e4m3_value((uint8_t)lo);
    double dhi = vo_e4m3_value((uint8_t)hi) - a;
    int code;
    if (dlo < dhi)
        code = lo;
    else if (dhi < dlo)
        code = hi;
    else
        code = (lo & 1) ? hi : lo; /* tie: the code whose mantissa LSB is 0 */
    return sign | (uint8_t)code;
}

VO_API void vo_e4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = vo_e4m3_encode(x[i]);
}

VO_API void vo_e4m3_value_array(const uint8_t* c, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = vo_e4m3_value(c[i]);
}

/* ------------------------------------------------------------------------ */
/* E2M1 codec (OCP MX FP4), from the format definition: sign bit 3, exponent  */
/* bits 2..1 (bias 1), mantissa bit 0; exponent field 0 is subnormal (m/2).   */
/* No infinities or NaN; the largest magnitude is 6.                          */
/* ------------------------------------------------------------------------ */
VO_API double vo_e2m1_value(uint8_t code) {
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double v = e == 0 ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return sign ? -v : v;
}

/* Nearest E2M1 value, ties to the even code, saturating to +-6. */
VO_API uint8_t vo_e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs((double)x);
    if (a >= 6.0) return sign | 0x7;
    int lo = 0; /* value(lo) <= a < value(lo + 1) */
    while (lo < 7 && vo_e2m1_value((uint8_t)(lo + 1)) <= a) ++lo;
    double dlo = a - vo_e2m1_value((uint8_t)lo);
    double dhi = vo_e2m1_value((uint8_t)(lo + 1)) - a;
    int code;
    if (dlo < dhi)
        code = lo;
    else if (dhi < dlo)
        code = lo + 1;
    else
        code = (lo & 1) ? lo + 1 : lo;
    return sign | (uint8_t)code;
}

VO_API void vo_e2m1_value_array(const uint8_t* c, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = vo_e2m1_value(c[i]);
}

VO_API void vo_e2m1_encode_array(const float* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = vo_e2m1_encode(x[i]);
}

/* One NVFP4 block of n <= 16 values: the UE4M3 scale s = E4M3(amax/6) (the
 * quotient in fp32), then each code E2M1(x * r) with r = 1/value(s) in fp32.
 * A zero scale gives zero codes. */
VO_API void vo_nvfp4_block(const float* x, int n, uint8_t* codes, uint8_t* scale) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i)
        if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
    uint8_t s = vo_e4m3_encode(amax / 6.0f);
    float sv = (float)vo_e4m3_value(s);
    *scale = s;
    if (sv == 0.0f) {
        for (int i = 0; i < n; ++i) codes[i] = 0;
        return;
    }
    float r = 1.0f / sv;
    for (int i = 0; i < n; ++i) codes[i] = vo_e2m1_encode(x[i] * r);
}

/* nblocks consecutive blocks of len values each */
VO_API void vo_nvfp4_block_array(const float* x, int64_t nblocks, int len, uint8_t* codes, uint8_t* scales) {
    for (int64_t b = 0; b < nblocks; ++b) vo_nvfp4_block(x + b * len, len, codes + b * len, scales + b);
}

/* ------------------------------------------------------------------------ */
/* ExpCast-FP8 [ChooseAI/ExpCast]: the E4M3 byte of a probability p is about  */
/* 8*log2(p) + 56, so a log2-domain score z maps straight to the byte        */
/* round(8z + 56 + beta) with one multiply-add.  Here 8z + 56 + beta is       */
/* A*s + Cb, where A*s is 8*log2(e)*score and Cb = 56 + beta - 8M is an        */
/* integer.  The exact value A*s + Cb is rounded once, ties to even, and      */
/* clamped below at 0.                                                        */
/* ------------------------------------------------------------------------ */
static double round_half_even_plus(double d, double cb) {
    /* rne(d + cb) for an exactly representable d and an integer cb, without
     * forming d + cb (which could round).  The fraction of d + cb is the
     * fraction of d; a tie goes to the even sum. */
    double fl = floor(d);
    double fr = d - fl; /* exact */
    double n;
    if (fr > 0.5)
        n = fl + 1.0;
    else if (fr < 0.5)
        n = fl;
    else
        n = (fmod(fl + cb, 2.0) == 0.0) ? fl : fl + 1.0;
    return n + cb;
}

VO_API uint8_t vo_expcast_byte(float A, float s, float cb) {
    double d = (double)A * (double)s; /* exact: 24 x 24 significant bits */
    double t = round_half_even_plus(d, (double)cb);
    if (!(t > 0.0)) return 0;
    if (t > 255.0) return 255; /* never reached for t <= 56 + beta <= 126 */
    return (uint8_t)t;
}

VO_API void vo_expcast_array(const float* A, const float* s, const float* cb, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = vo_expcast_byte(A[i], s[i], cb[i]);
}

/* ------------------------------------------------------------------------ */
/* k-means over one head's value tokens [ChooseAI/V-Smooth] (a lightweight  */
/* k-means) and [Clarity] (like value tokens share a cluster). Plain Lloyd. */
/* ------------------------------------------------------------------------ */
VO_API void vo_kmeans(const uint16_t* v, int n, int d, int C, int iters, int32_t* labels, double* cent) {
    double* sums = (double*)calloc((size_t)C * d, sizeof(double));
    int64_t* cnt = (int64_t*)calloc((size_t)C, sizeof(int64_t));
    double* vd = (double*)malloc(sizeof(double) * (size_t)n * d);
    for (size_t e = 0; e < (size_t)n * d; ++e) vd[e] = bf16_to_float(v[e]);
    for (int k = 0; k < C; ++k) {
        int64_t src = ((int64_t)k * n) / C;
        for (int c = 0; c < d; ++c) cent[(size_t)k * d + c] = vd[(size_t)src * d + c];
    }
    double* ct = (double*)malloc(sizeof(double) * (size_t)C * d); /* centroids, channel-major */
    for (int it = 0; it < iters; ++it) {
        for (int k = 0; k < C; ++k)
            for (int c = 0; c < d; ++c) ct[(size_t)c * C + k] = cent[(size_t)k * d + c];
        /* assignment: tokens are independent, so they are split over threads;
         * each token's distances are summed over channels in order */
#pragma omp parallel
        {
            double* dist = (double*)malloc(sizeof(double) * (size_t)C);
#pragma omp for schedule(static)
            for (int j = 0; j < n; ++j) {
                for (int k = 0; k < C; ++k) dist[k] = 0.0;
                for (int c = 0; c < d; ++c) {
                    const double x = vd[(size_t)j * d + c];
                    const double* row = ct + (size_t)c * C;
                    for (int k = 0; k < C; ++k) {
                        const double diff = x - row[k];
                        dist[k] += diff * diff;
                    }
                }
                int best = 0;
                for (int k = 1; k < C; ++k)
                    if (dist[k] < dist[best]) best = k; /* strict: ties keep the lowest k */
                labels[j] = best;
            }
            free(dist);
        }
        if (it == iters - 1) break;
        memset(sums, 0, sizeof(double) * (size_t)C * d);
        memset(cnt, 0, sizeof(int64_t) * (size_t)C);
        for (int j = 0; j < n; ++j) {
            cnt[labels[j]] += 1;
            for (int c = 0; c < d; ++c) sums[(size_t)labels[j] * d + c] += vd[(size_t)j * d + c];
        }
        for (int k = 0; k < C; ++k)
            if (cnt[k] > 0)
                for (int c = 0; c < d; ++c) cent[(size_t)k * d + c] = sums[(size_t)k * d + c] / (double)cnt[k];
    }
    free(ct);
    free(vd);
    free(sums);
    free(cnt);
}

/* Stable regroup: tokens ordered by cluster id, original order inside a
 * cluster.  perm[i] is the original index of the token at position i. */
VO_API void vo_stable_perm(const int32_t* labels, int n, int C, int32_t* perm) {
    int64_t* start = (int64_t*)calloc((size_t)C + 1, sizeof(int64_t));
    for (int j = 0; j < n; ++j) start[labels[j] + 1] += 1;
    for (int k = 0; k < C; ++k) start[k + 1] += start[k];
    for (int j = 0; j < n; ++j) perm[start[labels[j]]++] = j;
    free(start);
}

/* ------------------------------------------------------------------------ */
/* Q/K quantisation.  The pages only say Q and K go to 8 bits before QK^T     */
/* (chooseai.io news 7051, "一句话说清楚" and V-Smooth sections); this is the    */
/* per-token (Q) / per-block (K) amax reading.                               */
/* ------------------------------------------------------------------------ */
static void quant_rows(const uint16_t* x, const int32_t* rows, int nrows, int d, uint8_t* out, float* scale) {
    float amax = 0.0f;
    for (int r = 0; r < nrows; ++r)
        for (int c = 0; c < d; ++c) {
            float a = fabsf(bf16_to_float(x[(size_t)rows[r] * d + c]));
            if (a > amax) amax = a;
        }
    float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
    *scale = amax / 448.0f;
    for (int r = 0; r < nrows; ++r)
        for (int c = 0; c < d; ++c) {
            float y = bf16_to_float(x[(size_t)rows[r] * d + c]) * inv;
            out[(size_t)r * d + c] = vo_e4m3_encode(y);
        }
}

/* Q: one scale per token.  qhat [nrows*d], sq [nrows]. */
VO_API void vo_quant_q(const uint16_t* q, int nrows, int d, uint8_t* qhat, float* sq) {
    for (int i = 0; i < nrows; ++i) {
        int32_t row = i;
        quant_rows(q, &row, 1, d, qhat + (size_t)i * d, &sq[i]);
    }
}

/* K in regrouped order, one scale per block of bk tokens.  khat [T*bk*d]
 * (padding rows zero), ksc [T]. */
VO_API void vo_quant_k(const uint16_t* k, int n, int d, int bk, const int32_t* perm, uint8_t* khat, float* ksc) {
    int T = (n + bk - 1) / bk;
    memset(khat, 0, (size_t)T * bk * d);
    for (int b = 0; b < T; ++b) {
        int valid = (n - b * bk) < bk ? (n - b * bk) : bk;
        quant_rows(k, perm + (size_t)b * bk, valid, d, khat + (size_t)b * bk * d, &ksc[b]);
    }
}

/* V-Smooth [ChooseAI/V-Smooth], [Clarity], [MarkTechPost]: similar value tokens
 * share a block; the block mean is subtracted and kept in high precision
 * (fp32); the residual goes to E4M3 with one scale per channel.
 * smooth == 0 is plain per-channel FP8 V: identity order and zero means.
 * vhat [T*bk*d] token-major in regrouped order (padding rows zero),
 * vmu [T*d], vsc [d]. */
VO_API void vo_smooth_v(const uint16_t* v, int n, int d, int bk, const int32_t* perm, int smooth, uint8_t* vhat,
                        float* vmu, float* vsc) {
    int T = (n + bk - 1) / bk;
    float* amax = (float*)calloc((size_t)d, sizeof(float));
    float* inv = (float*)calloc((size_t)d, sizeof(float));
    memset(vhat, 0, (size_t)T * bk * d);
    for (int b = 0; b < T; ++b) {
        int valid = (n - b * bk) < bk ? (n - b * bk) : bk;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            if (smooth)
                for (int r = 0; r < valid; ++r) s += (double)bf16_to_float(v[(size_t)perm[b * bk + r] * d + c]);
            vmu[(size_t)b * d + c] = smooth ? (float)(s / (double)valid) : 0.0f;
        }
        for (int r = 0; r < valid; ++r)
            for (int c = 0; c < d; ++c) {
                float res = bf16_to_float(v[(size_t)perm[b * bk + r] * d + c]) - vmu[(size_t)b * d + c];
                if (fabsf(res) > amax[c]) amax[c] = fabsf(res);
            }
    }
    for (int c = 0; c < d; ++c) {
        vsc[c] = amax[c] > 0.0f ? amax[c] / 448.0f : 1.0f;
        inv[c] = amax[c] > 0.0f ? 448.0f / amax[c] : 0.0f;
    }
    for (int b = 0; b < T; ++b) {
        int valid = (n - b * bk) < bk ? (n - b * bk) : bk;
        for (int r = 0; r < valid; ++r)
            for (int c = 0; c < d; ++c) {
                float res = bf16_to_float(v[(size_t)perm[b * bk + r] * d + c]) - vmu[(size_t)b * d + c];
                vhat[((size_t)b * bk + r) * d + c] = vo_e4m3_encode(res * inv[c]);
            }
    }
    free(amax);
    free(inv);
}

/* The 4-bit residual [MarkTechPost] (per-channel scales, NVFP4 codes): the
 * same block means and residuals as vo_smooth_v; per channel one fp32 scale
 * s_c = amax_c/(6*448), y = r * (6*448/amax_c); then NVFP4 blocks of 16
 * consecutive tokens of a channel inside each hardware block (bk a multiple of
 * 16; padding tokens count as 0).
 * vq [T*bk*d] E2M1 codes token-major (padding rows zero), vgs [T*(bk/16)*d]
 * UE4M3 block scales ([T][bk/16][d]), vmu [T*d], vsc [d]. */
VO_API void vo_smooth_v_nvfp4(const uint16_t* v, int n, int d, int bk, const int32_t* perm, int smooth, uint8_t* vq,
                              uint8_t* vgs, float* vmu, float* vsc) {
    int T = (n + bk - 1) / bk;
    int G = bk / 16;
    float* amax = (float*)calloc((size_t)d, sizeof(float));
    float* inv = (float*)calloc((size_t)d, sizeof(float));
    float* y = (float*)malloc(sizeof(float) * (size_t)bk * d);
    float x[16];
    uint8_t codes[16];
    memset(vq, 0, (size_t)T * bk * d);
    for (int b = 0; b < T; ++b) {
        int valid = (n - b * bk) < bk ? (n - b * bk) : bk;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            if (smooth)
                for (int r = 0; r < valid; ++r) s += (double)bf16_to_float(v[(size_t)perm[b * bk + r] * d + c]);
            vmu[(size_t)b * d + c] = smooth ? (float)(s / (double)valid) : 0.0f;
        }
        for (int r = 0; r < valid; ++r)
            for (int c = 0; c < d; ++c) {
                float res = bf16_to_float(v[(size_t)perm[b * bk + r] * d + c]) - vmu[(size_t)b * d + c];
                if (fabsf(res) > amax[c]) amax[c] = fabsf(res);
            }
    }
    for (int c = 0; c < d; ++c) {
        vsc[c] = amax[c] > 0.0f ? amax[c] / 2688.0f : 1.0f;
        inv[c] = amax[c] > 0.0f ? 2688.0f / amax[c] : 0.0f;
    }
    for (int b = 0; b < T; ++b) {
        int valid = (n - b * bk) < bk ? (n - b * bk) : bk;
        for (int r = 0; r < bk; ++r)
            for (int c = 0; c < d; ++c) {
                float res = r < valid ? bf16_to_float(v[(size_t)perm[b * bk + r] * d + c]) - vmu[(size_t)b * d + c]
                                      : 0.0f;
                y[(size_t)r * d + c] = res * inv[c];
            }
        for (int g = 0; g < G; ++g)
            for (int c = 0; c < d; ++c) {
                for (int i = 0; i < 16; ++i) x[i] = y[(size_t)(16 * g + i) * d + c];
                vo_nvfp4_block(x, 16, codes, &vgs[((size_t)b * G + g) * d + c]);
                for (int i = 0; i < 16; ++i) vq[((size_t)b * bk + 16 * g + i) * d + c] = codes[i];
            }
    }
    free(amax);
    free(inv);
    free(y);
}

/* ------------------------------------------------------------------------ */
/* The quantised attention forward, replayed row by row in tile order.       */
/*                                                                            */
/* Inputs are values, so the same routine serves the quantised method and     */
/* the exact identity-quantiser check:                                        */
/*   qv [nrows*d], sq [nrows]       query values and per-row scale            */
/*   kv [T*bk*d], ksc [T]           key values (regrouped), per-block scale    */
/*   rv [T*bk*d], vmu [T*d], vsc[d] residual values, block means, channel     */
/*                                  scales: v = vmu_b + vsc * rv               */
/* kappa = 8*log2(e)/sqrt(d) (the caller passes its fp32 rounding).          */
/* exact == 0: the method -- fp32 scores, fp32 A = (kappa*sq)*sk, ExpCast     */
/*             bytes, p = E4M3 value of the byte.                             */
/* exact == 1: fp64 scores and A, p = 2^((t - 56)/8) with t unrounded.        */
/* rowmask (may be NULL): [nrows][T]; 0 drops key tile b for row i, as a     */
/*             block-sparse mask would (the tile takes no part in the row's    */
/*             max, weights or sums); a row with no tile left outputs 0.       */
/* pfmt == 1 (4-bit path, exact == 0): each 16-key block of a tile's P is     */
/*             re-coded to NVFP4 (vo_nvfp4_block on the E4M3 values; keys past */
/*             n count as 0) and p is the coded value.                         */
/* Output: out [nrows*d] in fp64 (before the final bf16 rounding), and, when   */
/* non-NULL, the final integer reference Mout and normaliser lout per row.    */
/* ------------------------------------------------------------------------ */
VO_API void vo_attn_emul(const double* qv, const float* sq, int nrows, const double* kv, const float* ksc,
                         const double* rv, const float* vmu, const float* vsc, int n, int d, int bk, double kappa,
                         int beta, int exact, int pfmt, const uint8_t* rowmask, double* out, double* Mout,
                         double* lout) {
    int T = (n + bk - 1) / bk;
    double* sc = (double*)malloc(sizeof(double) * (size_t)bk);
    double* p = (double*)malloc(sizeof(double) * (size_t)bk);
    double* ores = (double*)malloc(sizeof(double) * (size_t)d);
    double* omean = (double*)malloc(sizeof(double) * (size_t)d);
    float kappa32 = (float)kappa;
    for (int i = 0; i < nrows; ++i) {
        const double* q = qv + (size_t)i * d;
        double M = 0.0, l = 0.0;
        int first = 1;
        for (int c = 0; c < d; ++c) ores[c] = omean[c] = 0.0;
        float aq32 = kappa32 * sq[i];
        for (int b = 0; b < T; ++b) {
            if (rowmask && !rowmask[(size_t)i * T + b]) continue;
            int valid = (n - b * bk) < bk ? (n - b * bk) : bk;
            double A;
            if (exact)
                A = kappa * (double)sq[i] * (double)ksc[b];
            else
                A = (double)(aq32 * ksc[b]);
            /* scores of the valid keys of this tile */
            double mx = -INFINITY;
            for (int j = 0; j < valid; ++j) {
                const double* kr = kv + ((size_t)b * bk + j) * d;
                double s = 0.0;
                for (int c = 0; c < d; ++c) s += q[c] * kr[c];
                sc[j] = exact ? s : (double)(float)s;
                if (sc[j] > mx) mx = sc[j];
            }
            /* integer row reference, raised online */
            double x = exact ? A * mx : (double)((float)A * (float)mx);
            double Mc = ceil(x / 8.0);
            double Mnew = first ? Mc : (Mc > M ? Mc : M);
            if (!first && Mnew > M) {
                double f = ldexp(1.0, -(int)(Mnew - M));
                for (int c = 0; c < d; ++c) {
                    ores[c] *= f;
                    omean[c] *= f;
                }
                l *= f;
            }
            M = Mnew;
            first = 0;
            double cb = 56.0 + (double)beta - 8.0 * M;
            double lb = 0.0;
            for (int j = 0; j < valid; ++j) {
                if (exact) {
                    double t = A * sc[j] + cb;
                    p[j] = exp2((t - 56.0) / 8.0);
                } else {
                    p[j] = vo_e4m3_value(vo_expcast_byte((float)A, (float)sc[j], (float)cb));
                }
            }
            if (!exact && pfmt == 1) {
                float x[16];
                uint8_t codes[16], sc16;
                for (int g = 0; g < bk / 16; ++g) {
                    for (int i = 0; i < 16; ++i) x[i] = 16 * g + i < valid ? (float)p[16 * g + i] : 0.0f;
                    vo_nvfp4_block(x, 16, codes, &sc16);
                    for (int i = 0; i < 16 && 16 * g + i < valid; ++i)
                        p[16 * g + i] = vo_e4m3_value(sc16) * vo_e2m1_value(codes[i]);
                }
            }
            for (int j = 0; j < valid; ++j) lb += p[j];
            /* residual part through the quantised V, mean part as l_b * mu_b */
            for (int j = 0; j < valid; ++j) {
                const double* rr = rv + ((size_t)b * bk + j) * d;
                for (int c = 0; c < d; ++c) ores[c] += p[j] * rr[c];
            }
            for (int c = 0; c < d; ++c) omean[c] += lb * (double)vmu[(size_t)b * d + c];
            l += lb;
        }
        for (int c = 0; c < d; ++c) out[(size_t)i * d + c] = first ? 0.0 : ((double)vsc[c] * ores[c] + omean[c]) / l;
        if (Mout) Mout[i] = M;
        if (lout) lout[i] = l;
    }
    free(sc);
    free(p);
    free(ores);
    free(omean);
}

/* ------------------------------------------------------------------------ */
/* Exact attention: softmax(q k^T / sqrt(d)) v on the bf16 inputs widened to  */
/* fp64, non-causal (plain self-attention over one token sequence,           */
/* [RuntimeWire]).  rows [nrows] selects query rows.                          */
/* ------------------------------------------------------------------------ */
VO_API void vo_attn_exact(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* rows, int nrows,
                          int n, int d, double* out) {
    double* w = (double*)malloc(sizeof(double) * (size_t)n);
    double scale = 1.0 / sqrt((double)d);
    for (int i = 0; i < nrows; ++i) {
        const uint16_t* qr = q + (size_t)rows[i] * d;
        double mx = -INFINITY;
        for (int j = 0; j < n; ++j) {
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += (double)bf16_to_float(qr[c]) * (double)bf16_to_float(k[(size_t)j * d + c]);
            w[j] = s * scale;
            if (w[j] > mx) mx = w[j];
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) {
            w[j] = exp(w[j] - mx);
            l += w[j];
        }
        double* o = out + (size_t)i * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int j = 0; j < n; ++j)
            for (int c = 0; c < d; ++c) o[c] += w[j] * (double)bf16_to_float(v[(size_t)j * d + c]);
        for (int c = 0; c < d; ++c) o[c] /= l;
    }
    free(w);
}
