/*
 * vca_oracle.c -- plain, slow CPU oracle for VC-Attention-style FP8 attention.
 *
 * TEST INFRASTRUCTURE ONLY (see vca_oracle.h): used by the tests, the smoke
 * check and the benchmark's CPU-baseline leg, never by the product path.
 *
 * Sources (page titles; sections named where they have one):
 *   [VCA-news] "VC-Attention: Training-Free Low-Bit Attention Speeds Video
 *              Diffusion Up to 3.6x" -- V-Smooth and ExpCast-FP8 bullets.
 *   [VCA-mtp]  "Nunchux AI Introduces VC-Attention: A Training-Free Low-Bit
 *              Attention Kernel That Speeds Up Video Diffusion Transformers"
 *              -- Chinese section "V-Smooth 與 ExpCast-FP8" and the English
 *              abstract ("An E4M3 byte is already close to a logarithm...").
 *   [VCA-ru]   "VC-Attention" (aikraft.ru) -- section "Решение".
 *
 * Where the pages leave a step open, the reading taken is marked READING and
 * restated in the repository's design notes.
 */
#include "vca_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define VO_BLOCK 128

int vo_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ bf16 */

float vo_bf16_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to the nearest bf16 (8 significant bits), ties to even,
 * in one step (no intermediate float rounding). */
uint16_t vo_double_to_bf16_rne(double x) {
    if (isnan(x)) return 0x7FC0;
    if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
    double a = fabs(x);
    int e;
    frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
    int qexp = e - 8;             /* quantum of an 8-significant-bit number */
    if (qexp < -133) qexp = -133; /* bf16 subnormal quantum 2^-133 */
    double q = ldexp(a, -qexp);   /* exact (power-of-two scaling) */
    double r = nearbyint(q);      /* default rounding mode: ties to even */
    double y = ldexp(r, qexp);    /* exact */
    float f = (float)y;           /* exact: y has <= 8 significant bits */
    if (signbit(x)) f = -f;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);   /* exact: low 16 bits are zero (or inf) */
}

/* ------------------------------------------------------------------ E4M3 */

/* E4M3 decode from the format's definition: value = (-1)^s * 2^(E-7) * (1+M/8)
 * for E >= 1, (-1)^s * 2^-6 * (M/8) for E = 0, NaN for E=15,M=7.
 * ([VCA-mtp]: ExpCast reads this byte, as an integer, as ~8*log2(v)+56.) */
double vo_e4m3_decode(uint8_t code) {
    int s = code >> 7, E = (code >> 3) & 15, M = code & 7;
    double v;
    if (E == 15 && M == 7) return NAN;
    if (E == 0) v = ldexp((double)M, -9);
    else        v = ldexp(1.0 + M / 8.0, E - 7);
    return s ? -v : v;
}

/* Table of the 127 non-negative finite E4M3 values in code order (ascending). */
static double g_e4m3_pos[127];
static int g_e4m3_init = 0;
static void e4m3_table_init(void) {
    if (g_e4m3_init) return;
    for (int c = 0; c < 127; ++c) g_e4m3_pos[c] = vo_e4m3_decode((uint8_t)c);
    g_e4m3_init = 1;
}

/* Nearest E4M3 to x, ties to the even code, finite values saturated to +-448
 * (READING: saturating conversion; a NaN input gives 0x7F; negative values that
 * round to zero keep the sign, 0x80). */
uint8_t vo_e4m3_encode(float x) {
    e4m3_table_init();
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    /* binary search for the last code with value <= a */
    int lo = 0, hi = 126;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (g_e4m3_pos[mid] <= a) lo = mid; else hi = mid - 1;
    }
    int c = lo;
    if (c < 126) {
        double dlo = a - g_e4m3_pos[c], dhi = g_e4m3_pos[c + 1] - a;
        if (dhi < dlo || (dhi == dlo && ((c + 1) & 1) == 0)) c = c + 1;
    }
    return sign | (uint8_t)c;
}

void vo_e4m3_encode_array(const float* x, uint8_t* out, int64_t n) {
    e4m3_table_init();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = vo_e4m3_encode(x[i]);
}

/* --------------------------------------------------------------- ExpCast */

/* ExpCast-FP8 ([VCA-news] ExpCast-FP8 bullet; [VCA-mtp] abstract; [VCA-ru]
 * "Решение"): the E4M3 byte of p = 2^z is written straight from z with one
 * fused multiply-add, byte = 8*z + 56 + beta with beta = -0.35, instead of
 * computing 2^z in fp32 and casting.
 * READING: the FMA is fp32 fmaf(8, z, 55.65f); rounding to the byte is
 * round-to-nearest-even (the pages' 79.6% same-byte rate holds for RNE, not for
 * truncation); the byte is clamped to [0, 126] (0 = probability 0, 126 = 448,
 * 127 would be NaN); codes 1..7 are left as computed and decode as E4M3
 * subnormals (the "underflow tail"); z = NaN gives 0x7F. */
uint8_t vo_expcast(float z, int flags) {
    if (isnan(z)) return 0x7F;
    float addend = (flags & VO_PLANT_BETA0) ? 56.0f : 55.65f;
    float a = fmaf(8.0f, z, addend);
    float r = (flags & VO_PLANT_TRUNC) ? floorf(a) : rintf(a);
    if (r < 0.0f) r = 0.0f;
    if (r > 126.0f) r = 126.0f;
    return (uint8_t)r;
}

void vo_expcast_array(const float* z, uint8_t* out, int64_t n, int flags) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = vo_expcast(z[i], flags);
}

/* ------------------------------------------------------------- E2M1, NVFP4 */

/* E2M1, the element type of NVFP4 ("Accelerating Video Generation with GEMM
 * Quantization, Attention Quantization and Skip Softmax Attention in
 * TensorRT-LLM", table of quantisation formats): a sign bit, 2 exponent bits
 * with bias 1 and 1 mantissa bit; exponent field 0 holds 0 and the subnormal
 * 0.5; no infinities, no NaN; largest magnitude 6.  Bits 0..2 of a code hold
 * the magnitude, bit 3 the sign. */
double vo_e2m1_decode(uint8_t code) {
    int e = (code >> 1) & 3, m = code & 1;
    double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (code & 8) ? -mag : mag;
}

/* Nearest E2M1 value, ties to the even code, finite values saturating at +-6;
 * the sign is kept (a negative that rounds to 0 gives 0x8). */
uint8_t vo_e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 8 : 0;
    double a = fabs((double)x);
    uint8_t k = 0;
    for (; k < 7; ++k) {
        double mid = 0.5 * (vo_e2m1_decode(k) + vo_e2m1_decode((uint8_t)(k + 1)));
        if (a < mid || (a == mid && (k & 1) == 0)) break;
    }
    return sign | k;
}

/* NVFP4 (same table): E2M1 elements, one E4M3 scale per 16 consecutive
 * elements, one fp32 scale per tensor.  READING (the pages give the format,
 * not the rounding recipe): with the tensor scale G (fp32, > 0) a group's
 * scale is chosen so that its largest element lands on 6, and both quotients
 * are taken in fp32 as a kernel takes them:
 *   t = amax_g / (6 G);  sc = e4m3(t);  s = decode(sc)
 *   code_i = e2m1(x_i * (1 / (s G)))
 * (one rounding per fp32 product, quotient and reciprocal).  A group whose
 * scale decodes to 0 gets zero codes.  An element stands for G * s * e2m1(code).
 * Writes n codes (16 for a whole group), one nibble per byte; returns sc. */
static uint8_t nvfp4_group(const float* x, int n, float G, uint8_t* codes) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i)
        if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
    float t = amax / (6.0f * G);
    uint8_t sc = vo_e4m3_encode(t);
    float sg = (float)vo_e4m3_decode(sc) * G;
    float inv = sg > 0.0f ? 1.0f / sg : 0.0f;
    for (int i = 0; i < n; ++i) codes[i] = sg > 0.0f ? vo_e2m1_encode(x[i] * inv) : 0;
    return sc;
}

void vo_nvfp4_quantize(const float* x, int64_t n, float G, uint8_t* codes, uint8_t* scales) {
    e4m3_table_init();
    for (int64_t g = 0; g * 16 < n; ++g) {
        int len = n - g * 16 < 16 ? (int)(n - g * 16) : 16;
        scales[g] = nvfp4_group(x + g * 16, len, G, codes + g * 16);
    }
}

/* --------------------------------------------------------------- k-means */

/* Squared L2 distance in fp32, channel order 0..d-1, one fmaf per channel.
 * READING: the pages say only "lightweight k-means" ([VCA-ru] "Решение") /
 * "lightweight online clustering" ([VCA-news]); this fixed fp32 order makes
 * the assignment reproducible bit for bit. */
static float sqdist_f32(const float* v, const float* mu, int d) {
    float acc = 0.0f;
    for (int c = 0; c < d; ++c) {
        float t = v[c] - mu[c];
        acc = fmaf(t, t, acc);
    }
    return acc;
}

/* Assignment step: each token goes to the centroid at least squared distance;
 * ties go to the lowest cluster index. */
void vo_kmeans_assign(const float* v, int N, int d, const float* cent, int k,
                      int32_t* assign) {
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        const float* x = v + (int64_t)n * d;
        int best = 0;
        float bd = sqdist_f32(x, cent, d);
        for (int c = 1; c < k; ++c) {
            float dd = sqdist_f32(x, cent + (int64_t)c * d, d);
            if (dd < bd) { bd = dd; best = c; }
        }
        assign[n] = best;
    }
}

/* Update step: each centroid becomes the mean of its members.  READING: the
 * sum is taken exactly in 2^-24 fixed point (int64), so its value does not
 * depend on summation order; mean = (float)(sum / (count * 2^24)) with one
 * fp64 division; a cluster with no members keeps its previous centroid. */
void vo_kmeans_update(const float* v, int N, int d, const int32_t* assign, int k,
                      float* cent, int32_t* counts) {
    int64_t* sums = (int64_t*)calloc((size_t)k * d, sizeof(int64_t));
    for (int c = 0; c < k; ++c) counts[c] = 0;
    for (int n = 0; n < N; ++n) {
        int a = assign[n];
        counts[a] += 1;
        for (int ch = 0; ch < d; ++ch)
            sums[(int64_t)a * d + ch] += llrint((double)v[(int64_t)n * d + ch] * 16777216.0);
    }
    for (int c = 0; c < k; ++c) {
        if (counts[c] == 0) continue;
        double den = (double)counts[c] * 16777216.0;
        for (int ch = 0; ch < d; ++ch)
            cent[(int64_t)c * d + ch] = (float)((double)sums[(int64_t)c * d + ch] / den);
    }
    free(sums);
}

/* Lloyd k-means on one head's value tokens.  READING: features are the raw
 * value vectors; the initial centroid c is token floor(c*N/k) unless warm-start
 * centroids are given; `iters` rounds of (assign all, then update all); the
 * returned assignment is the one the final centroids are the means of. */
void vo_kmeans_head(const uint16_t* V, int N, int d, int k, int iters,
                    const float* init, float* cent, int32_t* assign, int32_t* counts) {
    float* v = (float*)malloc((size_t)N * d * sizeof(float));
    for (int64_t i = 0; i < (int64_t)N * d; ++i) v[i] = vo_bf16_to_float(V[i]);
    if (init) {
        memcpy(cent, init, (size_t)k * d * sizeof(float));
    } else {
        for (int c = 0; c < k; ++c) {
            int64_t src = ((int64_t)c * N) / k;
            memcpy(cent + (int64_t)c * d, v + src * d, (size_t)d * sizeof(float));
        }
    }
    for (int it = 0; it < iters; ++it) {
        vo_kmeans_assign(v, N, d, cent, k, assign);
        vo_kmeans_update(v, N, d, assign, k, cent, counts);
    }
    free(v);
}

/* --------------------------------------------------------------- permutation */

/* Tokens reordered by cluster, original order kept inside a cluster
 * ([VCA-mtp]: the block mean removes more energy "after sorting").
 * perm[new position] = original index. */
void vo_stable_perm(const int32_t* assign, int N, int k, int32_t* perm) {
    int64_t* off = (int64_t*)calloc((size_t)k + 1, sizeof(int64_t));
    for (int n = 0; n < N; ++n) off[assign[n] + 1] += 1;
    for (int c = 0; c < k; ++c) off[c + 1] += off[c];
    for (int n = 0; n < N; ++n) perm[off[assign[n]]++] = n;
    free(off);
}

/* --------------------------------------------------------------- quantise */

/* Smallest integer e with amax <= 448 * 2^e (0 for amax = 0), clamped to the
 * UE8M0 exponent range [-127, 127].  READING: the pages fix no V-residual scale
 * format; a power of two keeps the rescale exact. */
int vo_v_exponent(float amax) {
    if (!(amax > 0.0f)) return 0;
    int E;
    double f = frexp((double)amax, &E);   /* amax = f * 2^E, f in [0.5, 1) */
    /* 448 = 0.875 * 2^9, so amax <= 448*2^e  <=>  f * 2^(E-9-e) <= 0.875 */
    int e = (f <= 0.875) ? E - 9 : E - 8;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* Per-block symmetric E4M3 quantisation of 128 token rows (Q in original order,
 * K in permuted order): scale = amax/448 (fp32), codes = E4M3(x * (448/amax))
 * with saturation; an all-zero block gets scale 1 and zero codes. */
static void quant_rows_block(const float* x /* [nv][d] */, int nv, int d,
                             uint8_t* out /* [128][d] */, float* scale) {
    float amax = 0.0f;
    for (int i = 0; i < nv * d; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    memset(out, 0, (size_t)VO_BLOCK * d);
    if (!(amax > 0.0f)) { *scale = 1.0f; return; }
    *scale = amax / 448.0f;
    float inv = 448.0f / amax;
    for (int i = 0; i < nv * d; ++i) out[i] = vo_e4m3_encode(x[i] * inv);
}

/* The V block mean of V-Smooth: per channel, the exact fixed-point sum of the
 * block's nv values, one fp64 division, one rounding to bf16 (mean_out[d]);
 * xv [nv][d] is replaced in place by the fp32 residual v - mean.  Returns the
 * residual's largest magnitude. */
static float v_block_residual(float* xv, int nv, int d, uint16_t* mean_out) {
    float amax = 0.0f;
    for (int c = 0; c < d; ++c) {
        int64_t S = 0;
        for (int t = 0; t < nv; ++t) S += llrint((double)xv[t * d + c] * 16777216.0);
        double mean = (double)S / ((double)nv * 16777216.0);
        uint16_t mb = vo_double_to_bf16_rne(mean);
        mean_out[c] = mb;
        float mf = vo_bf16_to_float(mb);
        for (int t = 0; t < nv; ++t) {
            float r = xv[t * d + c] - mf;
            xv[t * d + c] = r;
            if (fabsf(r) > amax) amax = fabsf(r);
        }
    }
    return amax;
}

/* V-Smooth on one head ([VCA-news] V-Smooth bullet; [VCA-ru] "Решение";
 * [VCA-mtp] 0.125 bit per value element for the mean):
 *   K and V rows are gathered by the permutation; in each block of 128
 *   permuted tokens the per-channel mean of V is taken and stored (READING:
 *   exact fixed-point sum, one fp64 division, rounded once to bf16 -- 16 bits
 *   per (block, channel) = 0.125 bit per element); only the residual
 *   r = v - mean (fp32) is quantised to E4M3 with a power-of-two block scale;
 *   K (permuted) and Q (original order) get per-block fp32 scales. */
void vo_smooth_quantize_head(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const int32_t* perm, int N, int d,
                             uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                             uint8_t* VrT, int8_t* v_exp, uint16_t* v_mean) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    memset(VrT, 0, (size_t)d * Np);
#pragma omp parallel for schedule(dynamic)
    for (int b = 0; b < nb; ++b) {
        int n0 = b * VO_BLOCK;
        int nv = N - n0 < VO_BLOCK ? N - n0 : VO_BLOCK;
        float* xq = (float*)malloc((size_t)VO_BLOCK * d * sizeof(float));
        float* xk = (float*)malloc((size_t)VO_BLOCK * d * sizeof(float));
        float* xv = (float*)malloc((size_t)VO_BLOCK * d * sizeof(float));
        for (int t = 0; t < nv; ++t) {
            int64_t src = perm[n0 + t];
            for (int c = 0; c < d; ++c) {
                xq[t * d + c] = vo_bf16_to_float(Q[(int64_t)(n0 + t) * d + c]);
                xk[t * d + c] = vo_bf16_to_float(K[src * d + c]);
                xv[t * d + c] = vo_bf16_to_float(V[src * d + c]);
            }
        }
        quant_rows_block(xq, nv, d, Qq + (int64_t)n0 * d, &q_scale[b]);
        quant_rows_block(xk, nv, d, Kq + (int64_t)n0 * d, &k_scale[b]);
        float amax = v_block_residual(xv, nv, d, v_mean + (int64_t)b * d);
        int e = vo_v_exponent(amax);
        v_exp[b] = (int8_t)e;
        for (int c = 0; c < d; ++c)
            for (int t = 0; t < nv; ++t)
                VrT[(int64_t)c * Np + n0 + t] = vo_e4m3_encode(ldexpf(xv[t * d + c], -e));
        free(xq); free(xk); free(xv);
    }
}

/* A second reading of the V residual scale: one power-of-two exponent per head
 * (the smallest e with max|r| <= 448 * 2^e over the whole head) instead of one
 * per block.  E4M3 carries its own exponent, so coding every block with the
 * head's step changes only the elements that fall below the normal range.  Same
 * outputs as vo_smooth_quantize_head; v_exp[b] holds the head exponent for
 * every block. */
void vo_smooth_quantize_head_vhead(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                   const int32_t* perm, int N, int d,
                                   uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                                   uint8_t* VrT, int8_t* v_exp, uint16_t* v_mean) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    float* R = (float*)malloc((size_t)N * d * sizeof(float));   /* residuals, permuted order */
    float* bmax = (float*)malloc((size_t)nb * sizeof(float));
    memset(VrT, 0, (size_t)d * Np);
#pragma omp parallel for schedule(dynamic)
    for (int b = 0; b < nb; ++b) {
        int n0 = b * VO_BLOCK;
        int nv = N - n0 < VO_BLOCK ? N - n0 : VO_BLOCK;
        float* xq = (float*)malloc((size_t)VO_BLOCK * d * sizeof(float));
        float* xk = (float*)malloc((size_t)VO_BLOCK * d * sizeof(float));
        for (int t = 0; t < nv; ++t) {
            int64_t src = perm[n0 + t];
            for (int c = 0; c < d; ++c) {
                xq[t * d + c] = vo_bf16_to_float(Q[(int64_t)(n0 + t) * d + c]);
                xk[t * d + c] = vo_bf16_to_float(K[src * d + c]);
                R[(int64_t)(n0 + t) * d + c] = vo_bf16_to_float(V[src * d + c]);
            }
        }
        quant_rows_block(xq, nv, d, Qq + (int64_t)n0 * d, &q_scale[b]);
        quant_rows_block(xk, nv, d, Kq + (int64_t)n0 * d, &k_scale[b]);
        bmax[b] = v_block_residual(R + (int64_t)n0 * d, nv, d, v_mean + (int64_t)b * d);
        free(xq); free(xk);
    }
    float amax = 0.0f;
    for (int b = 0; b < nb; ++b)
        if (bmax[b] > amax) amax = bmax[b];
    int e = vo_v_exponent(amax);
    for (int b = 0; b < nb; ++b) v_exp[b] = (int8_t)e;
#pragma omp parallel for schedule(static)
    for (int c = 0; c < d; ++c)
        for (int j = 0; j < N; ++j)
            VrT[(int64_t)c * Np + j] = vo_e4m3_encode(ldexpf(R[(int64_t)j * d + c], -e));
    free(R);
    free(bmax);
}

/* The 4-bit V-Smooth variant ([VCA-mtp] abstract and Chinese section: a 4-bit
 * V-Smooth runs on workstation cards; ExpCast is 8-bit only because NVFP4 has
 * no single affine log-to-code map).  READING: the 4-bit change is confined to
 * the PV product -- Q and K are quantised exactly as in the 8-bit variant, the
 * V block means are the same bf16 means, and only the residual r = v - mean
 * moves from E4M3 to NVFP4, in groups of 16 consecutive permuted tokens of one
 * channel (the key dimension is the PV contraction dimension), with one tensor
 * scale per head: G = amax_head(|r|) / (6 * 448), G = 1 for an all-zero
 * residual.  Outputs besides the 8-bit ones:
 *   VrT4 [d][Np/2]: token j of channel c in byte c*Np/2 + j/2, low nibble for
 *                   even j; v_sc [d][Np/16]: E4M3 group scales; *v_gscale = G.
 * Padding tokens (j >= N) have zero codes; groups wholly past N zero scales. */
void vo_smooth_quantize_head_fp4(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                 const int32_t* perm, int N, int d,
                                 uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                                 uint8_t* VrT4, uint8_t* v_sc, float* v_gscale, uint16_t* v_mean) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    float* R = (float*)malloc((size_t)N * d * sizeof(float));   /* residuals, permuted order */
    float* bmax = (float*)malloc((size_t)nb * sizeof(float));
#pragma omp parallel for schedule(dynamic)
    for (int b = 0; b < nb; ++b) {
        int n0 = b * VO_BLOCK;
        int nv = N - n0 < VO_BLOCK ? N - n0 : VO_BLOCK;
        float* xq = (float*)malloc((size_t)VO_BLOCK * d * sizeof(float));
        float* xk = (float*)malloc((size_t)VO_BLOCK * d * sizeof(float));
        for (int t = 0; t < nv; ++t) {
            int64_t src = perm[n0 + t];
            for (int c = 0; c < d; ++c) {
                xq[t * d + c] = vo_bf16_to_float(Q[(int64_t)(n0 + t) * d + c]);
                xk[t * d + c] = vo_bf16_to_float(K[src * d + c]);
                R[(int64_t)(n0 + t) * d + c] = vo_bf16_to_float(V[src * d + c]);
            }
        }
        quant_rows_block(xq, nv, d, Qq + (int64_t)n0 * d, &q_scale[b]);
        quant_rows_block(xk, nv, d, Kq + (int64_t)n0 * d, &k_scale[b]);
        bmax[b] = v_block_residual(R + (int64_t)n0 * d, nv, d, v_mean + (int64_t)b * d);
        free(xq); free(xk);
    }
    float amax = 0.0f;
    for (int b = 0; b < nb; ++b)
        if (bmax[b] > amax) amax = bmax[b];
    float G = amax > 0.0f ? amax / 2688.0f : 1.0f;
    *v_gscale = G;
    memset(VrT4, 0, (size_t)d * (Np / 2));
    memset(v_sc, 0, (size_t)d * (Np / 16));
#pragma omp parallel for schedule(static)
    for (int c = 0; c < d; ++c) {
        float x[16];
        uint8_t codes[16];
        for (int j0 = 0; j0 < N; j0 += 16) {
            int n = N - j0 < 16 ? N - j0 : 16;
            for (int i = 0; i < n; ++i) x[i] = R[(int64_t)(j0 + i) * d + c];
            v_sc[(int64_t)c * (Np / 16) + j0 / 16] = nvfp4_group(x, n, G, codes);
            for (int i = 0; i < n; ++i) {
                int64_t j = j0 + i;
                VrT4[(int64_t)c * (Np / 2) + j / 2] |= (uint8_t)(codes[i] << (4 * (j & 1)));
            }
        }
    }
    free(R);
    free(bmax);
}

/* SAGE-style quantisation, the comparison recipe of "Accelerating Video
 * Generation with GEMM Quantization, Attention Quantization and Skip Softmax
 * Attention in TensorRT-LLM" (section "Quantized Attention": q_block_size 1,
 * k_block_size 16, v_block_size 1, FP8 V), with K smoothed by its channel
 * mean (SageAttention2's K smoothing, named there as the line of work
 * followed).  No reordering, no block means:
 *   k_mean[c]  = bf16(exact mean of K[:, c] over all N tokens) (fixed-point
 *                sum, one fp64 division, one rounding -- as the V block mean)
 *   K' = K - k_mean (fp32); Q and K' get one fp32 scale per group (1 token
 *   for Q, 16 tokens for K'): amax / 448, codes e4m3(x * (448 / amax));
 *   V gets one fp32 scale per channel over all N tokens, same formula;
 *   VcT[c][j] = code of V[j][c] (channel-major, padded to Np with 0).
 *   q_scale [Np], k_scale [Np/16], v_chscale [d]; an all-zero group has
 *   scale 1 and codes 0. */
static void quant_group(const float* x, int n, uint8_t* out, float* scale) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i)
        if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
    if (!(amax > 0.0f)) {
        *scale = 1.0f;
        memset(out, 0, (size_t)n);
        return;
    }
    *scale = amax / 448.0f;
    float inv = 448.0f / amax;
    for (int i = 0; i < n; ++i) out[i] = vo_e4m3_encode(x[i] * inv);
}

/* The INT8 form of the same per-group rule, the post's other qk_dtype (int8,
 * the one it uses): scale = amax / 127, code = rne(x * (127 / amax)) with the
 * product in fp32, a signed byte in [-127, 127]; an all-zero group has scale 1
 * and codes 0. */
static void quant_group_i8(const float* x, int n, int8_t* out, float* scale) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i)
        if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
    if (!(amax > 0.0f)) {
        *scale = 1.0f;
        memset(out, 0, (size_t)n);
        return;
    }
    *scale = amax / 127.0f;
    float inv = 127.0f / amax;
    for (int i = 0; i < n; ++i) {
        float r = nearbyintf(x[i] * inv);   /* round half to even (default mode) */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        out[i] = (int8_t)r;
    }
}

/* Q and K' groups coded as E4M3 (qk_i8 = 0, Qq/Kq uint8) or INT8 (qk_i8 = 1,
 * Qq/Kq int8); V, k_mean and the layouts are the same in both. */
static void sage_quantize(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int N, int d, void* Qq,
                          float* q_scale, void* Kq, float* k_scale, uint8_t* VcT, float* v_chscale,
                          uint16_t* k_mean, int qk_i8) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    memset(Qq, 0, (size_t)Np * d);
    memset(Kq, 0, (size_t)Np * d);
    memset(VcT, 0, (size_t)Np * d);
    for (int64_t j = 0; j < Np; ++j) q_scale[j] = 1.0f;
    for (int64_t g = 0; g < Np / 16; ++g) k_scale[g] = 1.0f;
    float* x = (float*)malloc((size_t)16 * d * sizeof(float));
    for (int c = 0; c < d; ++c) {
        int64_t S = 0;
        for (int j = 0; j < N; ++j) S += llrint((double)vo_bf16_to_float(K[(int64_t)j * d + c]) * 16777216.0);
        k_mean[c] = vo_double_to_bf16_rne((double)S / ((double)N * 16777216.0));
    }
    for (int j = 0; j < N; ++j) {
        for (int c = 0; c < d; ++c) x[c] = vo_bf16_to_float(Q[(int64_t)j * d + c]);
        if (qk_i8)
            quant_group_i8(x, d, (int8_t*)Qq + (int64_t)j * d, &q_scale[j]);
        else
            quant_group(x, d, (uint8_t*)Qq + (int64_t)j * d, &q_scale[j]);
    }
    for (int g = 0; g * 16 < N; ++g) {
        int n = N - g * 16 < 16 ? N - g * 16 : 16;
        for (int t = 0; t < n; ++t)
            for (int c = 0; c < d; ++c)
                x[t * d + c] = vo_bf16_to_float(K[(int64_t)(g * 16 + t) * d + c]) - vo_bf16_to_float(k_mean[c]);
        if (qk_i8)
            quant_group_i8(x, n * d, (int8_t*)Kq + (int64_t)g * 16 * d, &k_scale[g]);
        else
            quant_group(x, n * d, (uint8_t*)Kq + (int64_t)g * 16 * d, &k_scale[g]);
    }
    float* col = (float*)malloc((size_t)N * sizeof(float));
    uint8_t* cc = (uint8_t*)malloc((size_t)N);
    for (int c = 0; c < d; ++c) {
        for (int j = 0; j < N; ++j) col[j] = vo_bf16_to_float(V[(int64_t)j * d + c]);
        quant_group(col, N, cc, &v_chscale[c]);
        memcpy(VcT + (int64_t)c * Np, cc, (size_t)N);
    }
    free(x);
    free(col);
    free(cc);
}

void vo_sage_quantize_head(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int N, int d,
                           uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                           uint8_t* VcT, float* v_chscale, uint16_t* k_mean) {
    sage_quantize(Q, K, V, N, d, Qq, q_scale, Kq, k_scale, VcT, v_chscale, k_mean, 0);
}

void vo_sage_quantize_head_i8(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int N, int d,
                              int8_t* Qq, float* q_scale, int8_t* Kq, float* k_scale,
                              uint8_t* VcT, float* v_chscale, uint16_t* k_mean) {
    sage_quantize(Q, K, V, N, d, Qq, q_scale, Kq, k_scale, VcT, v_chscale, k_mean, 1);
}

/* --------------------------------------------------------------- attention */

/* The ExpCast max grid: m = phi + n with integer n and phi = 0.65/8, so that
 * 8*(z - m) + 55.65 = 8*z + 55 - 8*n.  READING: snapping the row maximum to
 * this grid makes any two maxima differ by whole octaves, so the probability
 * codes computed against a running maximum equal the final ones shifted by a
 * multiple of 8 (an exact power-of-two rescale). */
#define VO_PHI (0.65 / 8.0)

/* READING: probabilities are encoded 4 octaves above the reference, i.e. the
 * byte written is ExpCast of z - m + 4: a maximum equal to the reference lands
 * on codes 80..88 (p between 8 and 16) instead of 48..56.  This fixed
 * power-of-two pre-scale cancels in the normalisation; it moves the E4M3
 * underflow tail 4 octaves further from the maximum.  The reference may lag
 * the running maximum by up to VO_LAG = 4 octaves (codes up to 120 < 126). */
#define VO_HEADROOM 4
#define VO_LAG 4

/* One query row of the same-algorithm attention ([VCA-news] V-Smooth and
 * ExpCast-FP8 bullets: the block mean is restored from the row sums that
 * online softmax keeps).  Operands are decoded values in fp64:
 *   q[d] and its block scale qs; kh[N][d], ks[N] (permuted keys and their
 *   block scales); rh[N][d] residual codes decoded; vexp[nb]; mu[nb][d].
 * Key blocks are visited in order, as online softmax does:
 *   s_j = q.k_j;  z_j = s_j*qs*ks_j*scale*log2(e)
 *   n_b = ceil(max_{j in b} z_j - phi)      (block maximum on the phi grid)
 *   the reference n is set by the first block and moves up to n_b only when
 *   n_b > n + VO_LAG; the accumulators are then scaled by 2^(n_old - n_b)
 *   p_j = decode(clamp(rne(8 z_j + 55 + 8*VO_HEADROOM - 8 n), 0, 126))
 *   l_b = sum_{j in b} p_j
 *   acc += 2^vexp_b sum_{j in b} p_j r_j + l_b mu_b;  L += l_b
 *   O = acc / L.
 * READING: the pages name online softmax but not its rescale rule; this one
 * (a reference that lags the running maximum by at most VO_LAG octaves) keeps
 * every code <= 56 + 8*(VO_HEADROOM + VO_LAG) = 120 < 126. */
/* Internal flag: the 4-bit variant's probabilities (see p_nvfp4_block). */
#define VO_P_NVFP4 (1 << 16)

/* READING: the probabilities of the 4-bit variant are bounded by
 * 2^(VO_HEADROOM + VO_LAG) = 256 by the reference rule, so their NVFP4 tensor
 * scale is the fixed power of two 2^-3 (the bound lands on a group scale of
 * 341 <= 448 with no pass over the data, and a power of two cancels exactly
 * against the row sum). */
#define VO_P_GSCALE 0.125f

/* NVFP4 quantisation of one key block of a row's probabilities, in place
 * (the 4-bit variant; ExpCast does not apply to 4 bits, so p is computed as
 * an exponential, rounded once to fp32, then quantised in groups of 16 keys
 * with tensor scale VO_P_GSCALE; the row sum then adds the dequantised values,
 * as the PV product does). */
static void p_nvfp4_block(double* pb, int n, int flags) {
    int gsz = (flags & VO_PLANT_P_GROUP32) ? 32 : 16;
    float x[32];
    uint8_t codes[32];
    for (int g0 = 0; g0 < n; g0 += gsz) {
        int len = n - g0 < gsz ? n - g0 : gsz;
        for (int i = 0; i < len; ++i) x[i] = (float)pb[g0 + i];
        uint8_t sc = nvfp4_group(x, len, VO_P_GSCALE, codes);
        double sg = vo_e4m3_decode(sc) * (double)VO_P_GSCALE;
        for (int i = 0; i < len; ++i) pb[g0 + i] = sg * vo_e2m1_decode(codes[i]);
    }
}

static void attn_row(const double* q, double qs, const double* kh, const double* ks,
                     const double* rh, const int* vexp, const double* mu, int N, int d,
                     double softmax_scale, int flags, double skip_log2, double* O, double* lse,
                     double* lblk, uint8_t* codes, int32_t* nref,
                     double* z /* scratch [N] */, double* acc /* [d] */) {
    const double log2e = 1.4426950408889634074;
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    double zall = -INFINITY;
    for (int j = 0; j < N; ++j) {
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += q[c] * kh[(int64_t)j * d + c];
        z[j] = s * qs * ks[j] * softmax_scale * log2e;
        if (z[j] > zall) zall = z[j];
    }
    const double headroom = (flags & VO_NO_HEADROOM) ? 0.0 : (double)VO_HEADROOM;
    for (int c = 0; c < d; ++c) acc[c] = 0.0;
    double ltot = 0.0, n = 0.0, zrun = -INFINITY;
    /* READING (second mode, VO_GLOBAL_MAX): the reference is the row maximum
     * over all keys snapped to the phi grid, fixed for the whole row -- the
     * plain form of a max-subtracted softmax, no online rescale. */
    if (flags & VO_GLOBAL_MAX) n = ceil(zall - VO_PHI);
    for (int b = 0; b < nb; ++b) {
        int j0 = b * VO_BLOCK, j1 = j0 + VO_BLOCK < N ? j0 + VO_BLOCK : N;
        double zmax = -INFINITY;
        for (int j = j0; j < j1; ++j)
            if (z[j] > zmax) zmax = z[j];
        /* Skip Softmax (BLASST): the block is negligible for this row when
         * exp(block max - running max) < lambda, i.e. in log2 units
         * zmax - zrun < log2(lambda); it then adds nothing (no probabilities,
         * no PV, zero row sum).  skip_log2 = -inf disables the rule.  A
         * rejected block lies below the running maximum, which the reference
         * trails by at most VO_LAG octaves, so it could not move the reference. */
        if (zmax > zrun) zrun = zmax;
        if (b > 0 && zmax - zrun < skip_log2) {
            if (lblk) lblk[b] = 0.0;
            if (codes) memset(codes + j0, 0, (size_t)(j1 - j0));
            if (nref) nref[b] = (int32_t)n;
            continue;
        }
        double nblk = ceil(zmax - VO_PHI);
        if (flags & VO_GLOBAL_MAX) {
            /* the reference is fixed */
        } else if (b == 0) {
            n = nblk;
        } else if (nblk > n + VO_LAG) {
            double sc = (flags & VO_PLANT_NO_RESCALE) ? 1.0 : exp2(n - nblk);   /* exact power of two */
            for (int c = 0; c < d; ++c) acc[c] *= sc;
            ltot *= sc;
            if (lblk)
                for (int b2 = 0; b2 < b; ++b2) lblk[b2] *= sc;
            n = nblk;
        }
        double lb = 0.0;
        double pv[512], pb[VO_BLOCK];
        for (int c = 0; c < d; ++c) pv[c] = 0.0;
        for (int j = j0; j < j1; ++j) {
            double p;
            if (flags & (VO_EXACT_EXP | VO_P_NVFP4)) {
                p = exp2(z[j] - (n + VO_PHI) + headroom);
            } else {
                /* = 8(z - m) + 55.65 + 8*headroom with m = n + phi */
                double x = 8.0 * z[j] + 55.0 - 8.0 * n + 8.0 * headroom;
                if (flags & VO_PLANT_BETA0) x += 0.35;
                double r = (flags & VO_PLANT_TRUNC) ? floor(x) : nearbyint(x);
                if (r < 0.0) r = 0.0;
                if (r > 126.0) r = 126.0;
                p = vo_e4m3_decode((uint8_t)r);
                if (codes) codes[j] = (uint8_t)r;
            }
            pb[j - j0] = p;
        }
        if ((flags & VO_P_NVFP4) && !(flags & VO_IDENTITY_QUANT)) p_nvfp4_block(pb, j1 - j0, flags);
        for (int j = j0; j < j1; ++j) {
            double p = pb[j - j0];
            lb += p;
            for (int c = 0; c < d; ++c) pv[c] += p * rh[(int64_t)j * d + c];
        }
        double sc = ldexp(1.0, vexp[b]);
        for (int c = 0; c < d; ++c) {
            acc[c] += sc * pv[c];
            if (!(flags & VO_PLANT_NO_MEAN)) acc[c] += lb * mu[(int64_t)b * d + c];
        }
        if (lblk) lblk[b] = lb;
        if (nref) nref[b] = (int32_t)n;
        ltot += lb;
    }
    for (int c = 0; c < d; ++c) O[c] = acc[c] / ltot;
    if (lse) *lse = log(2.0) * ((n + VO_PHI - headroom) + log2(ltot));
}

static void attn_rows(const double* qh, const double* qs_row, const double* kh,
                      const double* ks, const double* rh, const int* vexp,
                      const double* mu, int N, int d, double softmax_scale,
                      const int32_t* rows, int nrows, int flags, double skip_log2, double* O,
                      double* lse, double* lblk, uint8_t* codes, int32_t* nref) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
#pragma omp parallel
    {
        double* z = (double*)malloc((size_t)N * sizeof(double));
        double* acc = (double*)malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < nrows; ++r) {
            int i = rows[r];
            attn_row(qh + (int64_t)i * d, qs_row[i], kh, ks, rh, vexp, mu, N, d,
                     softmax_scale, flags, skip_log2, O + (int64_t)r * d, lse ? &lse[r] : NULL,
                     lblk ? lblk + (int64_t)r * nb : NULL, codes ? codes + (int64_t)r * N : NULL,
                     nref ? nref + (int64_t)r * nb : NULL, z, acc);
        }
        free(z);
        free(acc);
    }
}

static double skip_log2_of(double lambda) { return lambda > 0.0 ? log2(lambda) : -INFINITY; }

void vo_attention_head(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                       const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                       const uint16_t* v_mean, int N, int d, double softmax_scale,
                       const int32_t* rows, int nrows, int flags,
                       double* O, double* lse, double* lblk) {
    vo_attention_head_skip(Qq, q_scale, Kq, k_scale, VrT, v_exp, v_mean, N, d, softmax_scale, rows, nrows,
                           flags, 0.0, O, lse, lblk);
}

void vo_attention_head_skip(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                            const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                            const uint16_t* v_mean, int N, int d, double softmax_scale,
                            const int32_t* rows, int nrows, int flags, double skip_lambda,
                            double* O, double* lse, double* lblk) {
    vo_attention_head_ex(Qq, q_scale, Kq, k_scale, VrT, v_exp, v_mean, N, d, softmax_scale, rows, nrows, flags,
                         skip_lambda, O, lse, lblk, NULL, NULL);
}

void vo_attention_head_ex(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                          const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                          const uint16_t* v_mean, int N, int d, double softmax_scale,
                          const int32_t* rows, int nrows, int flags, double skip_lambda,
                          double* O, double* lse, double* lblk, uint8_t* codes, int32_t* nref) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    double* qh = (double*)malloc((size_t)N * d * sizeof(double));
    double* kh = (double*)malloc((size_t)N * d * sizeof(double));
    double* rh = (double*)malloc((size_t)N * d * sizeof(double));
    double* qs = (double*)malloc((size_t)N * sizeof(double));
    double* ks = (double*)malloc((size_t)N * sizeof(double));
    double* mu = (double*)malloc((size_t)nb * d * sizeof(double));
    int* ve = (int*)malloc((size_t)nb * sizeof(int));
    for (int j = 0; j < N; ++j) {
        qs[j] = q_scale[j / VO_BLOCK];
        ks[j] = k_scale[j / VO_BLOCK];
        for (int c = 0; c < d; ++c) {
            qh[(int64_t)j * d + c] = vo_e4m3_decode(Qq[(int64_t)j * d + c]);
            kh[(int64_t)j * d + c] = vo_e4m3_decode(Kq[(int64_t)j * d + c]);
            rh[(int64_t)j * d + c] = vo_e4m3_decode(VrT[(int64_t)c * Np + j]);
        }
    }
    for (int b = 0; b < nb; ++b) {
        ve[b] = v_exp[b];
        for (int c = 0; c < d; ++c) mu[(int64_t)b * d + c] = vo_bf16_to_float(v_mean[(int64_t)b * d + c]);
    }
    attn_rows(qh, qs, kh, ks, rh, ve, mu, N, d, softmax_scale, rows, nrows, flags, skip_log2_of(skip_lambda), O,
              lse, lblk, codes, nref);
    free(qh); free(kh); free(rh); free(qs); free(ks); free(mu); free(ve);
}

/* Attention on SAGE-style operands: the same row algorithm (ExpCast codes,
 * online reference) with per-token Q scales, per-16-key K scales, no V block
 * exponents or means, and output channel c multiplied by v_chscale[c]. */
static void sage_attention(const void* Qq, const float* q_scale, const void* Kq, const float* k_scale,
                           const uint8_t* VcT, const float* v_chscale, int N, int d, double softmax_scale,
                           const int32_t* rows, int nrows, int flags, double* O, double* lse, int qk_i8) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    double* qh = (double*)malloc((size_t)N * d * sizeof(double));
    double* kh = (double*)malloc((size_t)N * d * sizeof(double));
    double* rh = (double*)malloc((size_t)N * d * sizeof(double));
    double* qs = (double*)malloc((size_t)N * sizeof(double));
    double* ks = (double*)malloc((size_t)N * sizeof(double));
    double* mu = (double*)calloc((size_t)nb * d, sizeof(double));
    int* ve = (int*)calloc((size_t)nb, sizeof(int));
    for (int j = 0; j < N; ++j) {
        qs[j] = q_scale[j];
        ks[j] = k_scale[j / 16];
        for (int c = 0; c < d; ++c) {
            int64_t e = (int64_t)j * d + c;
            qh[e] = qk_i8 ? (double)((const int8_t*)Qq)[e] : vo_e4m3_decode(((const uint8_t*)Qq)[e]);
            kh[e] = qk_i8 ? (double)((const int8_t*)Kq)[e] : vo_e4m3_decode(((const uint8_t*)Kq)[e]);
            rh[e] = vo_e4m3_decode(VcT[(int64_t)c * Np + j]);
        }
    }
    attn_rows(qh, qs, kh, ks, rh, ve, mu, N, d, softmax_scale, rows, nrows, flags, -INFINITY, O, lse, NULL, NULL,
              NULL);
    for (int r = 0; r < nrows; ++r)
        for (int c = 0; c < d; ++c) O[(int64_t)r * d + c] *= v_chscale[c];
    free(qh); free(kh); free(rh); free(qs); free(ks); free(mu); free(ve);
}

void vo_attention_head_sage(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                            const float* k_scale, const uint8_t* VcT, const float* v_chscale,
                            int N, int d, double softmax_scale, const int32_t* rows, int nrows,
                            int flags, double* O, double* lse) {
    sage_attention(Qq, q_scale, Kq, k_scale, VcT, v_chscale, N, d, softmax_scale, rows, nrows, flags, O, lse, 0);
}

/* The same on INT8 Q and K' codes (vo_sage_quantize_head_i8): the code values
 * are the integers themselves, so q.k is exact; z, the codes and the rest of
 * the row algorithm are those of vo_attention_head_sage. */
void vo_attention_head_sage_i8(const int8_t* Qq, const float* q_scale, const int8_t* Kq,
                               const float* k_scale, const uint8_t* VcT, const float* v_chscale,
                               int N, int d, double softmax_scale, const int32_t* rows, int nrows,
                               int flags, double* O, double* lse) {
    sage_attention(Qq, q_scale, Kq, k_scale, VcT, v_chscale, N, d, softmax_scale, rows, nrows, flags, O, lse, 1);
}

/* The 4-bit variant's probability step on its own: n <= 128 consecutive keys
 * of one row (a key block), p[] the fp64 probabilities relative to the
 * reference; out[] the dequantised NVFP4 values the row sum and PV use. */
void vo_p_nvfp4(const double* p, int n, int flags, double* out) {
    for (int i = 0; i < n; ++i) out[i] = p[i];
    p_nvfp4_block(out, n, flags);
}

/* Attention of the 4-bit variant: the 8-bit row algorithm (online reference,
 * mean restore from the row sums) with NVFP4 probabilities (p_nvfp4_block)
 * and the NVFP4 V residual of vo_smooth_quantize_head_fp4, dequantised as
 * G * s * e2m1(code). */
void vo_attention_head_fp4(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                           const float* k_scale, const uint8_t* VrT4, const uint8_t* v_sc,
                           float v_gscale, const uint16_t* v_mean, int N, int d, double softmax_scale,
                           const int32_t* rows, int nrows, int flags, double* O, double* lse) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    double* qh = (double*)malloc((size_t)N * d * sizeof(double));
    double* kh = (double*)malloc((size_t)N * d * sizeof(double));
    double* rh = (double*)malloc((size_t)N * d * sizeof(double));
    double* qs = (double*)malloc((size_t)N * sizeof(double));
    double* ks = (double*)malloc((size_t)N * sizeof(double));
    double* mu = (double*)malloc((size_t)nb * d * sizeof(double));
    int* ve = (int*)calloc((size_t)nb, sizeof(int));
    for (int j = 0; j < N; ++j) {
        qs[j] = q_scale[j / VO_BLOCK];
        ks[j] = k_scale[j / VO_BLOCK];
        for (int c = 0; c < d; ++c) {
            qh[(int64_t)j * d + c] = vo_e4m3_decode(Qq[(int64_t)j * d + c]);
            kh[(int64_t)j * d + c] = vo_e4m3_decode(Kq[(int64_t)j * d + c]);
            uint8_t byte = VrT4[(int64_t)c * (Np / 2) + j / 2];
            int hi = (j & 1) ^ ((flags & VO_PLANT_NIBBLE) ? 1 : 0);
            uint8_t code = hi ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
            double s = vo_e4m3_decode(v_sc[(int64_t)c * (Np / 16) + j / 16]);
            rh[(int64_t)j * d + c] = (double)v_gscale * s * vo_e2m1_decode(code);
        }
    }
    for (int b = 0; b < nb; ++b)
        for (int c = 0; c < d; ++c) mu[(int64_t)b * d + c] = vo_bf16_to_float(v_mean[(int64_t)b * d + c]);
    attn_rows(qh, qs, kh, ks, rh, ve, mu, N, d, softmax_scale, rows, nrows, flags | VO_P_NVFP4, -INFINITY, O,
              lse, NULL, NULL, NULL);
    free(qh); free(kh); free(rh); free(qs); free(ks); free(mu); free(ve);
}

/* The 4-bit variant straight from bf16 Q/K/V and a permutation; with
 * VO_IDENTITY_QUANT no quantiser rounds (operands exact, exact fp64 block means,
 * exact probabilities), which must give exact softmax attention. */
void vo_attention_head_fp4_bf16(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                const int32_t* perm, int N, int d, double softmax_scale,
                                const int32_t* rows, int nrows, int flags, double* O) {
    if (flags & VO_IDENTITY_QUANT) {
        vo_attention_head_bf16_skip(Q, K, V, perm, N, d, softmax_scale, rows, nrows, flags | VO_P_NVFP4, 0.0, O);
        return;
    }
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    uint8_t* Qq = (uint8_t*)malloc((size_t)Np * d);
    uint8_t* Kq = (uint8_t*)malloc((size_t)Np * d);
    uint8_t* VrT4 = (uint8_t*)malloc((size_t)d * (Np / 2));
    uint8_t* vsc = (uint8_t*)malloc((size_t)d * (Np / 16));
    float* qsc = (float*)malloc((size_t)nb * sizeof(float));
    float* ksc = (float*)malloc((size_t)nb * sizeof(float));
    uint16_t* vm = (uint16_t*)malloc((size_t)nb * d * sizeof(uint16_t));
    float G = 1.0f;
    vo_smooth_quantize_head_fp4(Q, K, V, perm, N, d, Qq, qsc, Kq, ksc, VrT4, vsc, &G, vm);
    vo_attention_head_fp4(Qq, qsc, Kq, ksc, VrT4, vsc, G, vm, N, d, softmax_scale, rows, nrows, flags, O, NULL);
    free(Qq); free(Kq); free(VrT4); free(vsc); free(qsc); free(ksc); free(vm);
}

void vo_attention_head_bf16(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                            const int32_t* perm, int N, int d, double softmax_scale,
                            const int32_t* rows, int nrows, int flags, double* O) {
    vo_attention_head_bf16_skip(Q, K, V, perm, N, d, softmax_scale, rows, nrows, flags, 0.0, O);
}

void vo_attention_head_bf16_skip(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                 const int32_t* perm, int N, int d, double softmax_scale,
                                 const int32_t* rows, int nrows, int flags, double skip_lambda, double* O) {
    int nb = (N + VO_BLOCK - 1) / VO_BLOCK;
    int64_t Np = (int64_t)nb * VO_BLOCK;
    if (!(flags & VO_IDENTITY_QUANT)) {
        uint8_t* Qq = (uint8_t*)malloc((size_t)Np * d);
        uint8_t* Kq = (uint8_t*)malloc((size_t)Np * d);
        uint8_t* VrT = (uint8_t*)malloc((size_t)Np * d);
        float* qsc = (float*)malloc((size_t)nb * sizeof(float));
        float* ksc = (float*)malloc((size_t)nb * sizeof(float));
        int8_t* ve = (int8_t*)malloc((size_t)nb);
        uint16_t* vm = (uint16_t*)malloc((size_t)nb * d * sizeof(uint16_t));
        vo_smooth_quantize_head(Q, K, V, perm, N, d, Qq, qsc, Kq, ksc, VrT, ve, vm);
        vo_attention_head_skip(Qq, qsc, Kq, ksc, VrT, ve, vm, N, d, softmax_scale, rows, nrows,
                               flags, skip_lambda, O, NULL, NULL);
        free(Qq); free(Kq); free(VrT); free(qsc); free(ksc); free(ve); free(vm);
        return;
    }
    /* Identity quantisers: operands kept exactly, block means exact in fp64. */
    double* qh = (double*)malloc((size_t)N * d * sizeof(double));
    double* kh = (double*)malloc((size_t)N * d * sizeof(double));
    double* rh = (double*)malloc((size_t)N * d * sizeof(double));
    double* ones = (double*)malloc((size_t)N * sizeof(double));
    double* mu = (double*)malloc((size_t)nb * d * sizeof(double));
    int* ve = (int*)calloc((size_t)nb, sizeof(int));
    for (int j = 0; j < N; ++j) {
        ones[j] = 1.0;
        for (int c = 0; c < d; ++c) {
            qh[(int64_t)j * d + c] = vo_bf16_to_float(Q[(int64_t)j * d + c]);
            kh[(int64_t)j * d + c] = vo_bf16_to_float(K[(int64_t)perm[j] * d + c]);
            rh[(int64_t)j * d + c] = vo_bf16_to_float(V[(int64_t)perm[j] * d + c]);
        }
    }
    for (int b = 0; b < nb; ++b) {
        int j0 = b * VO_BLOCK, j1 = j0 + VO_BLOCK < N ? j0 + VO_BLOCK : N;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int j = j0; j < j1; ++j) s += rh[(int64_t)j * d + c];
            double m = s / (j1 - j0);
            mu[(int64_t)b * d + c] = m;
            for (int j = j0; j < j1; ++j) rh[(int64_t)j * d + c] -= m;
        }
    }
    attn_rows(qh, ones, kh, ones, rh, ve, mu, N, d, softmax_scale, rows, nrows, flags,
              skip_log2_of(skip_lambda), O, NULL, NULL, NULL, NULL);
    free(qh); free(kh); free(rh); free(ones); free(mu); free(ve);
}

/* Exact softmax attention in fp64, two passes (max, then sum) per row. */
void vo_exact_attention_head(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             int N, int d, double softmax_scale,
                             const int32_t* rows, int nrows, double* O) {
    double* kd = (double*)malloc((size_t)N * d * sizeof(double));
    double* vd = (double*)malloc((size_t)N * d * sizeof(double));
    for (int64_t i = 0; i < (int64_t)N * d; ++i) {
        kd[i] = vo_bf16_to_float(K[i]);
        vd[i] = vo_bf16_to_float(V[i]);
    }
#pragma omp parallel
    {
        double* a = (double*)malloc((size_t)N * sizeof(double));
        double* q = (double*)malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < nrows; ++r) {
            int i = rows[r];
            for (int c = 0; c < d; ++c) q[c] = vo_bf16_to_float(Q[(int64_t)i * d + c]);
            double m = -INFINITY;
            for (int j = 0; j < N; ++j) {
                double s = 0.0;
                for (int c = 0; c < d; ++c) s += q[c] * kd[(int64_t)j * d + c];
                a[j] = s * softmax_scale;
                if (a[j] > m) m = a[j];
            }
            double l = 0.0;
            double* o = O + (int64_t)r * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int j = 0; j < N; ++j) {
                double p = exp(a[j] - m);
                l += p;
                for (int c = 0; c < d; ++c) o[c] += p * vd[(int64_t)j * d + c];
            }
            for (int c = 0; c < d; ++c) o[c] /= l;
        }
        free(a);
        free(q);
    }
    free(kd);
    free(vd);
}
