/*
 * vca_oracle.h -- plain, slow CPU oracle for VC-Attention-style FP8 attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this
 * library: only the test suite, the package's smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library; it is written from the method's description on these pages:
 *
 *   [VCA-news] "VC-Attention: Training-Free Low-Bit Attention Speeds Video
 *              Diffusion Up to 3.6x" (agihunt.info news summary).
 *   [VCA-mtp]  "Nunchux AI Introduces VC-Attention: A Training-Free Low-Bit
 *              Attention Kernel That Speeds Up Video Diffusion Transformers"
 *              (MarkTechPost abstract, mirrored with a Chinese summary on
 *              yifor-blog; sections "V-Smooth 與 ExpCast-FP8" and the English
 *              abstract).
 *   [VCA-ru]   "VC-Attention" (aikraft.ru news), section "Решение:
 *              VC-Attention без дообучения".
 *   [TRT-blog] "Accelerating Video Generation with GEMM Quantization, Attention
 *              Quantization and Skip Softmax Attention in TensorRT-LLM": the
 *              Skip Softmax rule, the SAGE-style comparison recipe and the NVFP4
 *              format (E2M1 elements, E4M3 scale per 16, fp32 per tensor).
 *
 * Arithmetic: fp64 wherever the method does not fix a precision; fp32 with
 * explicit fmaf() where the method (or a stated reading of it) fixes fp32.
 * Build with -O2 -ffp-contract=off and no fast-math.
 *
 * bf16 tensors are passed as their raw uint16 bit patterns.
 * All per-head arrays are row-major: [N][d] for token rows, [d][Np] for the
 * transposed V residual, [nb][d] for block means.
 */
#ifndef VCA_ORACLE_H
#define VCA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- flags for vo_attention_* (reductions and planted mistakes) ---- */
#define VO_EXACT_EXP       1   /* p = 2^(z - m) in fp64 instead of ExpCast codes     */
#define VO_IDENTITY_QUANT  2   /* bf16 path only: no E4M3 rounding, exact fp64 means  */
#define VO_PLANT_TRUNC     64  /* planted mistake: ExpCast truncates instead of RNE  */
#define VO_PLANT_NO_MEAN   128 /* planted mistake: drop the rowsum*mean restore term */
#define VO_PLANT_BETA0     256 /* planted mistake: addend 56 instead of 56 + beta    */
#define VO_PLANT_NO_RESCALE 512 /* planted mistake: reference moves without rescaling */
#define VO_PLANT_NIBBLE    1024 /* planted mistake (4-bit): V nibbles read high first  */
#define VO_PLANT_P_GROUP32 2048 /* planted mistake (4-bit): P groups of 32 keys       */
#define VO_GLOBAL_MAX      4096 /* second reading: fixed reference = snapped row max  */
#define VO_NO_HEADROOM     8192 /* codes written at the reference (no 4-octave pre-scale) */

/* E4M3 (OCP FP8: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities, NaN = S.1111.111, largest finite 448). */
double  vo_e4m3_decode(uint8_t code);
uint8_t vo_e4m3_encode(float x);
void    vo_e4m3_encode_array(const float* x, uint8_t* out, int64_t n);

/* ExpCast-FP8 on a log2-domain, max-subtracted score z. */
uint8_t vo_expcast(float z, int flags);
void    vo_expcast_array(const float* z, uint8_t* out, int64_t n, int flags);

/* E2M1 (NVFP4 element: sign, 2 exponent bits with bias 1, 1 mantissa bit;
 * magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6), nearest with ties to even, saturating. */
double  vo_e2m1_decode(uint8_t code);
uint8_t vo_e2m1_encode(float x);
/* NVFP4 quantisation of x[n] in groups of 16 with tensor scale G: codes[n] (one
 * nibble per byte) and scales[ceil(n/16)] E4M3 codes. */
void    vo_nvfp4_quantize(const float* x, int64_t n, float G, uint8_t* codes, uint8_t* scales);

/* bf16 helpers. */
float    vo_bf16_to_float(uint16_t b);
uint16_t vo_double_to_bf16_rne(double x);

/* k-means over the value tokens of one head. */
void vo_kmeans_assign(const float* v, int N, int d, const float* cent, int k,
                      int32_t* assign);
void vo_kmeans_update(const float* v, int N, int d, const int32_t* assign, int k,
                      float* cent, int32_t* counts);
void vo_kmeans_head(const uint16_t* V, int N, int d, int k, int iters,
                    const float* init /* nullable [k][d] */, float* cent /* [k][d] */,
                    int32_t* assign /* [N] */, int32_t* counts /* [k] */);

/* Stable counting sort by cluster id: perm[new] = old. */
void vo_stable_perm(const int32_t* assign, int N, int k, int32_t* perm);

/* V-Smooth quantisation of one head (block = 128 tokens, Np = 128*ceil(N/128)). */
int  vo_v_exponent(float amax);
void vo_smooth_quantize_head(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             const int32_t* perm, int N, int d,
                             uint8_t* Qq /* [Np][d] */, float* q_scale /* [nb] */,
                             uint8_t* Kq /* [Np][d] */, float* k_scale /* [nb] */,
                             uint8_t* VrT /* [d][Np] */, int8_t* v_exp /* [nb] */,
                             uint16_t* v_mean /* [nb][d] */);

/* Same-algorithm attention for selected query rows of one head, from the
 * quantised operands.  O is [nrows][d] fp64, lse [nrows] (nullable),
 * lblk [nrows][nb] per-block row sums (nullable). */
void vo_attention_head(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                       const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                       const uint16_t* v_mean, int N, int d, double softmax_scale,
                       const int32_t* rows, int nrows, int flags,
                       double* O, double* lse, double* lblk);

/* Same, with Skip Softmax (BLASST, "Accelerating Video Generation with GEMM
 * Quantization, Attention Quantization and Skip Softmax Attention in
 * TensorRT-LLM", section "Sparse Attention with Skip Softmax"): key block j is
 * dropped for row i when exp(block max - running max) < skip_lambda (scores in
 * natural-log units; the running max includes block j).  skip_lambda = 0 is
 * the plain algorithm; 0 <= skip_lambda < 1. */
void vo_attention_head_skip(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                            const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                            const uint16_t* v_mean, int N, int d, double softmax_scale,
                            const int32_t* rows, int nrows, int flags, double skip_lambda,
                            double* O, double* lse, double* lblk);

/* Same, also returning what each row coded: codes [nrows][N] (the E4M3 byte
 * written for each permuted key, against the reference in effect when its
 * block was visited; 0 for dropped blocks) and nref [nrows][nb] (that
 * reference's integer n, the maximum being n + 0.65/8).  Both nullable. */
void vo_attention_head_ex(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                          const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                          const uint16_t* v_mean, int N, int d, double softmax_scale,
                          const int32_t* rows, int nrows, int flags, double skip_lambda,
                          double* O, double* lse, double* lblk, uint8_t* codes, int32_t* nref);

/* SAGE-style comparison recipe (TensorRT-LLM video post, section "Quantized
 * Attention": per-token Q scales, one K scale per 16 tokens after K-mean
 * smoothing, per-channel FP8 V; no reordering, no block means).
 * q_scale [Np], k_scale [Np/16], VcT [d][Np], v_chscale [d], k_mean [d] bf16. */
void vo_sage_quantize_head(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int N, int d,
                           uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                           uint8_t* VcT, float* v_chscale, uint16_t* k_mean);
void vo_attention_head_sage(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                            const float* k_scale, const uint8_t* VcT, const float* v_chscale,
                            int N, int d, double softmax_scale, const int32_t* rows, int nrows,
                            int flags, double* O, double* lse);
/* The post's INT8 qk_dtype: Q and K' groups as signed bytes, scale amax/127,
 * code rne(x * (127/amax)) in fp32; V, k_mean and layouts as above. */
void vo_sage_quantize_head_i8(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int N, int d,
                              int8_t* Qq, float* q_scale, int8_t* Kq, float* k_scale,
                              uint8_t* VcT, float* v_chscale, uint16_t* k_mean);
void vo_attention_head_sage_i8(const int8_t* Qq, const float* q_scale, const int8_t* Kq,
                               const float* k_scale, const uint8_t* VcT, const float* v_chscale,
                               int N, int d, double softmax_scale, const int32_t* rows, int nrows,
                               int flags, double* O, double* lse);

/* A second reading of the V residual scale: one exponent per head (v_exp[b] all
 * equal to it); everything else as vo_smooth_quantize_head. */
void vo_smooth_quantize_head_vhead(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                   const int32_t* perm, int N, int d,
                                   uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                                   uint8_t* VrT, int8_t* v_exp, uint16_t* v_mean);

/* The 4-bit V-Smooth variant ("Nunchux AI Introduces VC-Attention...",
 * abstract: 4-bit V-Smooth on workstation cards; ExpCast is 8-bit only).
 * Q, K, v_mean as in vo_smooth_quantize_head; the V residual in NVFP4:
 * VrT4 [d][Np/2] (low nibble = even token), v_sc [d][Np/16] E4M3 group
 * scales, *v_gscale the head's fp32 tensor scale. */
void vo_smooth_quantize_head_fp4(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                 const int32_t* perm, int N, int d,
                                 uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                                 uint8_t* VrT4, uint8_t* v_sc, float* v_gscale, uint16_t* v_mean);
/* Attention on those operands with NVFP4 probabilities (16-key groups, tensor
 * scale 2^-3); O [nrows][d] fp64, lse [nrows] nullable. */
void vo_attention_head_fp4(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                           const float* k_scale, const uint8_t* VrT4, const uint8_t* v_sc,
                           float v_gscale, const uint16_t* v_mean, int N, int d, double softmax_scale,
                           const int32_t* rows, int nrows, int flags, double* O, double* lse);
/* Its probability step alone: n <= 128 keys of one row, out = dequantised. */
void vo_p_nvfp4(const double* p, int n, int flags, double* out);
void vo_attention_head_fp4_bf16(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                const int32_t* perm, int N, int d, double softmax_scale,
                                const int32_t* rows, int nrows, int flags, double* O);

/* Same algorithm, straight from bf16 Q/K/V and a permutation; with
 * VO_IDENTITY_QUANT the quantisers are the identity (for reductions). */
void vo_attention_head_bf16(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                            const int32_t* perm, int N, int d, double softmax_scale,
                            const int32_t* rows, int nrows, int flags, double* O);
void vo_attention_head_bf16_skip(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                 const int32_t* perm, int N, int d, double softmax_scale,
                                 const int32_t* rows, int nrows, int flags, double skip_lambda, double* O);

/* Exact fp64 softmax(Q K^T * scale) V for selected rows of one head. */
void vo_exact_attention_head(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                             int N, int d, double softmax_scale,
                             const int32_t* rows, int nrows, double* O);

int vo_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
