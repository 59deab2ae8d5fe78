/*
 * vca.h -- C ABI of libvca.so: VC-Attention-style FP8 self-attention forward
 * for video diffusion-transformer token sequences, on B200 (sm_100a).
 *
 * The method (no code is published; described on these pages):
 *   [VCA-news] "VC-Attention: Training-Free Low-Bit Attention Speeds Video
 *              Diffusion Up to 3.6x" (agihunt.info): V-Smooth bullet (reorder
 *              value tokens by lightweight online clustering, quantise only the
 *              residual after the block mean, restore the mean from the online
 *              softmax row sums) and ExpCast-FP8 bullet (score -> E4M3
 *              probability code with one fused multiply-add).
 *   [VCA-mtp]  "Nunchux AI Introduces VC-Attention: A Training-Free Low-Bit
 *              Attention Kernel That Speeds Up Video Diffusion Transformers"
 *              (MarkTechPost abstract): byte ~ 8 log2(v) + 56, beta = -0.35,
 *              0.125 bit per value element for the mean, block sorting.
 *   [VCA-ru]   "VC-Attention" (aikraft.ru), section "Решение": k-means
 *              grouping, mean stored exactly, one FMA per probability byte.
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers owned by the caller, contiguous,
 *    16-byte aligned (VCA_ERR_INVALID otherwise).  The library allocates no
 *    device memory; scratch space is the caller's workspace `ws` of at least
 *    the size the matching *_workspace_size() returns.  The first 16 bytes of
 *    every workspace are the device status word; zero the workspace once after
 *    allocating it (vca_reset_status does this).
 *  - bf16 tensors are passed as uint16_t bit patterns (vca_bf16).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; 0 = legacy default).
 *    The return value reports argument and launch errors only; errors found on
 *    the device (a bounded wait that ran out, non-finite input) are recorded
 *    in the workspace status word and returned by vca_check_status().
 *  - Layouts: B batch, H heads, N tokens, d = 128 head channels,
 *    nb = ceil(N/128) blocks of 128 tokens, Np = 128*nb.  Q/K/V/O are
 *    [B][H][N][d] row-major.
 *  - Thread safety: calls are independent; two calls that share a workspace
 *    must not run concurrently on the GPU.
 */
#ifndef VCA_H
#define VCA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t vca_bf16;
typedef struct CUstream_st* vca_stream_t; /* same type as cudaStream_t */

#define VCA_OK 0
#define VCA_ERR_INVALID (-1)     /* null pointer, bad shape or alignment        */
#define VCA_ERR_UNSUPPORTED (-2) /* d != 128, block != 128, k or N out of range */
#define VCA_ERR_CUDA (-3)        /* a CUDA launch / runtime call failed         */
#define VCA_ERR_TIMEOUT (-4)     /* a device-side bounded wait ran out          */
#define VCA_ERR_NONFINITE (-5)   /* an input held inf/NaN (prep kernels)        */
#define VCA_ERR_WORKSPACE (-6)   /* workspace missing or smaller than required  */

#define VCA_HEAD_DIM 128
#define VCA_BLOCK 128
#define VCA_MAX_CLUSTERS 64

/* ------------------------------------------------------------------ status */

/* Bytes of the status word at the start of every workspace. */
size_t vca_status_bytes(void);

/* Zeroes the status word of `ws` (asynchronously on `stream`). */
int vca_reset_status(void* ws, vca_stream_t stream);

/* Synchronises `stream`, returns the first device-side error recorded in `ws`
 * since the last reset (VCA_OK if none) and clears it.  If `where`/`info` are
 * non-null they receive the kernel's location tag and detail. */
int vca_check_status(void* ws, vca_stream_t stream, int* where, int* info);

/* Message for the most recent failing call made by this host thread. */
const char* vca_last_error(void);

/* Device-side wait limit in nanoseconds for every bounded wait (default
 * 2e9).  Process-wide; takes effect for launches made after the call. */
void vca_set_wait_limit_ns(uint64_t ns);

/* Self-test of the bounded-wait path: launches one block that waits on an
 * mbarrier no thread ever arrives on, with a limit of `limit_ns`; the wait
 * runs out and VCA_ERR_TIMEOUT is recorded in `ws` (read it with
 * vca_check_status).  It faults nothing and returns in ~limit_ns. */
int vca_debug_wait_timeout(void* ws, uint64_t limit_ns, vca_stream_t stream);

/* ------------------------------------------------------------------ ExpCast */

/* ExpCast-FP8 reference map ([VCA-news] ExpCast-FP8 bullet; [VCA-mtp]: an
 * E4M3 byte read as an integer is ~8 log2(v) + 56, beta = -0.35).
 * For each of the n fp32 log2-domain, max-subtracted scores z[i]:
 *   codes[i] = clamp(rne(fmaf(8, z[i], 55.65f)), 0, 126)   (E4M3 byte of ~2^z)
 * with z = -inf -> 0 and z = NaN -> 0x7F.  z: n floats; codes: n bytes. */
int vca_expcast_ref(const float* z, uint8_t* codes, int64_t n, vca_stream_t stream);

/* E4M3 encoder used by the prep kernels: out[i] = e4m3(x[i]), round to nearest
 * even, finite values saturated to +-448 (hardware cvt ... satfinite).
 * x: n floats; out: n bytes. */
int vca_e4m3_encode(const float* x, uint8_t* out, int64_t n, vca_stream_t stream);

/* ------------------------------------------------------------------ V-Smooth */

size_t vca_cluster_permute_workspace_size(int B, int H, int N, int k);

/* V-Smooth grouping ([VCA-news]: value tokens reordered by lightweight online
 * clustering; [VCA-ru] "Решение": k-means groups similar tokens into blocks;
 * [VCA-mtp]: block means remove most energy after sorting).
 * Per (b, h) independently, Lloyd k-means on the value vectors:
 *   init: centroid c = V[floor(c*N/k)], or init_centroids [B][H][k][d] if
 *         non-null (warm start, e.g. from an earlier denoising step);
 *   iters rounds of: assign each token to the nearest centroid (fp32 squared
 *   distance accumulated with one fma per channel in channel order, ties to the
 *   lowest index), then centroid = exact mean of its members (2^-24 fixed-point
 *   sum, one fp64 division; an empty cluster keeps its centroid).
 * Then a stable counting sort by cluster gives perm[new] = old index.
 *   V          [B][H][N][d] bf16        (in)
 *   centroids  [B][H][k][d] fp32        (out)
 *   assign     [B][H][N] int32          (out, the assignment of the last round)
 *   perm       [B][H][N] int32          (out)
 * 1 <= k <= VCA_MAX_CLUSTERS, 1 <= iters <= 64, |V| < 2^20: a value outside
 * that range records VCA_ERR_INVALID (VCA_ERR_NONFINITE for inf/NaN) in the
 * workspace status word (vca_check_status), as does a device wait that runs
 * out (VCA_ERR_TIMEOUT).  All pointers 16-byte aligned, else VCA_ERR_INVALID.
 * The assignment evaluates the distance above only for the centroids that a
 * tensor-core estimate with a proven error bound cannot rule out; the result
 * is the full scan's, bit for bit. */
int vca_cluster_permute(const vca_bf16* V, int B, int H, int N, int d, int k, int iters,
                        const float* init_centroids, float* centroids, int32_t* assign,
                        int32_t* perm, void* ws, size_t ws_bytes, vca_stream_t stream);

/* Same grouping as vca_cluster_permute for callers that cannot allocate device
 * memory when they call it (for example a plugin inside an engine that owns the
 * whole GPU memory budget, or an enqueue path that must not risk the device-wide
 * synchronisation cudaMalloc can cause).  The pages have no counterpart: this is
 * a library convenience.  Identical arguments and results, minus the workspace:
 * scratch is one fixed array of VCA_NOALLOC_SCRATCH_BYTES inside the library,
 * held on every GPU that loads the library until the process exits.
 *  - Shapes whose workspace (vca_cluster_permute_workspace_size) exceeds that
 *    size are rejected with VCA_ERR_UNSUPPORTED; nothing is allocated, ever.
 *  - Every call looks up the array's device address with the caller's device
 *    current (a lookup, no allocation).
 *  - Every call uses the same array: calls whose work overlaps on the GPU race.
 *    Issue them on one stream, or serialise them.
 *  - The return value reports argument and launch errors only.  The input
 *    check the kernels make on the device (|V| >= 2^20 or non-finite values,
 *    which the exact sums cannot take) lands in a status word inside the array
 *    that no call returns: validate V beforehand, or use vca_cluster_permute,
 *    whose workspace status vca_check_status reads. */
#define VCA_NOALLOC_SCRATCH_BYTES (8u << 20)
int vca_cluster_permute_noalloc(const vca_bf16* V, int B, int H, int N, int d, int k, int iters,
                                const float* init_centroids, float* centroids, int32_t* assign,
                                int32_t* perm, vca_stream_t stream);

/* Denoising-schedule reuse of the grouping ([VCA-mtp], abstract and section
 * "V-Smooth 與 ExpCast-FP8": grouping runs only in the first 25 % of the
 * denoising steps and each permutation is reused across 4 adjacent steps, which
 * amortises the grouping to 3-4 % of attention time).  Host function, no GPU
 * work: returns 1 when step `step` (0-based) of a `total_steps`-step run should
 * regroup -- call vca_cluster_permute, warm-started from the centroids of the
 * previous grouping -- and 0 when it should keep the last permutation;
 * VCA_ERR_INVALID for step < 0, total_steps < 1, step >= total_steps,
 * reuse < 1 or group_fraction outside (0, 1].
 * Reading of the pages: a step regroups iff it is step 0, or
 * step < group_fraction * total_steps and step is a multiple of `reuse`
 * (defaults 0.25 and 4).  Quantisation (vca_smooth_quantize_qkv) runs at every
 * step, since Q, K and V change every step. */
int vca_schedule_regroup(int step, int total_steps, int reuse, float group_fraction);

size_t vca_smooth_quantize_workspace_size(int B, int H, int N);

/* V-Smooth quantisation ([VCA-news] V-Smooth bullet; [VCA-ru] "Решение": the
 * block mean is subtracted and stored exactly, only the residual is quantised;
 * [VCA-mtp]: 0.125 bit per value element for the mean).
 * Per (b, h) and block of 128 permuted tokens (the tail block holds N mod 128):
 *   K and V rows are gathered by perm; Q keeps the original order.
 *   v_mean[b][c]  = bf16(exact mean of V over the block's tokens)
 *   residual r    = V - v_mean (fp32);  v_exp[b] = smallest e with
 *                   max|r| <= 448 * 2^e (0 if r == 0), clamped to [-127, 127]
 *   VrT[c][j]     = e4m3(r * 2^-e)   (transposed: channel-major, Np tokens)
 *   Q/K blocks:   scale = max|x| / 448 (fp32), codes = e4m3(x * (448/max|x|))
 *                 (an all-zero block: scale 1, codes 0)
 *   e4m3() rounds to nearest even and saturates at +-448; padding (N..Np) is 0.
 * Outputs (all device):
 *   Qq [B][H][Np][d] u8, q_scale [B][H][nb] f32, Kq [B][H][Np][d] u8 (permuted),
 *   k_scale [B][H][nb] f32, VrT [B][H][d][Np] u8 (permuted), v_exp [B][H][nb] i8,
 *   v_mean [B][H][nb][d] bf16.
 * block must be 128.  Non-finite or |x| >= 2^20 inputs record
 * VCA_ERR_NONFINITE in the status word. */
int vca_smooth_quantize_qkv(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V,
                            const int32_t* perm, int B, int H, int N, int d, int block,
                            uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                            uint8_t* VrT, int8_t* v_exp, vca_bf16* v_mean, void* ws,
                            size_t ws_bytes, vca_stream_t stream);

/* ------------------------------------------------------------------ attention */

/* 4-bit V-Smooth quantisation ([VCA-mtp] abstract: the 4-bit V-Smooth of the
 * workstation parts; NVFP4 per [TRT-blog], table of quantisation formats:
 * E2M1 elements, one E4M3 scale per 16 elements, one fp32 scale per tensor).
 * Q, K, q_scale, k_scale and v_mean are exactly those of
 * vca_smooth_quantize_qkv; only the V residual r = V - v_mean changes, to NVFP4
 * in groups of 16 consecutive permuted tokens of one channel:
 *   v_gscale[b][h] = G = max|r| over the head / (6 * 448)  (1 if r == 0)
 *   group scale    sc = e4m3(max|r_group| / (6 G))
 *   codes          e2m1(r * (1 / (decode(sc) * G)))   (nearest, ties to the
 *                  even code, saturating at +-6; sign in bit 3)
 * every product, quotient and reciprocal rounded once in fp32; a group whose
 * scale decodes to 0 has zero codes.  Layouts per (b, h):
 *   VrT4 [d][Np/2] u8: token j of channel c in byte c*Np/2 + j/2, low nibble
 *        for even j; v_sc [d][Np/16] u8 E4M3 group scales; v_gscale fp32.
 * Padding tokens have zero codes, groups wholly past N zero scales.  Q, K, V,
 * Qq, Kq, VrT4 and v_sc 16-byte aligned; the workspace (status word and one
 * maximum per head) of vca_smooth_quantize_fp4_workspace_size() bytes.  Same
 * errors as vca_smooth_quantize_qkv. */
size_t vca_smooth_quantize_fp4_workspace_size(int B, int H, int N);
int vca_smooth_quantize_qkv_fp4(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V,
                                const int32_t* perm, int B, int H, int N, int d, uint8_t* Qq,
                                float* q_scale, uint8_t* Kq, float* k_scale, uint8_t* VrT4,
                                uint8_t* v_sc, float* v_gscale, vca_bf16* v_mean, void* ws,
                                size_t ws_bytes, vca_stream_t stream);

size_t vca_attention_workspace_size(int B, int H, int N);

/* ExpCast-FP8 attention forward, non-causal self-attention ([VCA-news]:
 * low-bit QK^T and PV, ExpCast-FP8 softmax, mean restored from the row sums
 * online softmax keeps).  For each query row i (original order) of head (b,h),
 * visiting the key blocks b = 0..nb-1 in (permuted) order:
 *   z_ij  = (Qq_i . Kq_j) * q_scale * k_scale * softmax_scale * log2(e)
 *   n_b   = ceil(max_{j in b} z_ij - phi), phi = 0.65/8 (block max on the grid)
 *   n     = reference: n_0 at the first block; it moves up to n_b only when
 *           n_b > n + 4, and everything accumulated so far is then scaled by
 *           the exact power of two 2^(n_old - n_b)
 *   p_ij  = E4M3 value of clamp(rne(8 z_ij + 55 + 32 - 8 n), 0, 126)
 *           (ExpCast-FP8 of the probability relative to n + phi, pre-scaled by
 *           2^4; every code stays <= 120)
 *   l_ib  = sum of p_ij over key block b
 *   O_i   = (sum_b 2^v_exp[b] sum_{j in b} p_ij VrT[:, j] + sum_b l_ib v_mean[b])
 *           / sum_b l_ib          -> O [B][H][N][d] bf16 (round to nearest even)
 *   lse_i = ln 2 * (n + phi - 4 + log2 sum_b l_ib)    (optional, [B][H][N] fp32)
 * Inputs are the outputs of vca_smooth_quantize_qkv; |z| must stay below 2^18.
 * The workspace needs only the status word (vca_attention_workspace_size). */
int vca_attention_fwd(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                      const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                      const vca_bf16* v_mean, int B, int H, int N, int d, float softmax_scale,
                      vca_bf16* O, float* lse, void* ws, size_t ws_bytes, vca_stream_t stream);

/* Attention of the 4-bit V-Smooth variant ([VCA-mtp] abstract: 4-bit V-Smooth;
 * ExpCast is 8-bit only, so the probabilities are exponentials quantised to
 * NVFP4; [TRT-blog] formats table: NVFP4 = E2M1 elements, one E4M3 scale per 16
 * elements, one fp32 scale per tensor).  Inputs are the outputs of
 * vca_smooth_quantize_qkv_fp4 (Qq, q_scale, Kq, k_scale as the 8-bit prep; VrT4
 * [B][H][d][Np/2] E2M1 codes, low nibble = even token; v_sc [B][H][d][Np/16]
 * E4M3 group scales, 8-byte aligned; v_gscale [B][H] fp32 head scales G).
 * z, the reference n and its rescale rule are those of vca_attention_fwd; then
 * for each row and key block, per 16 keys g:
 *   p_j  = 2^(z_ij - n - phi + 4) in fp32
 *   sc_g = e4m3(max_{j in g} p_j / 0.75), s_g = 2^-3 decode(sc_g)
 *   p^_j = s_g e2m1(p_j * (1 / s_g))       (one fp32 rounding per step)
 *   l_ib = sum of p^_j over key block b
 *   O_i  = (sum_j p^_j G s_v e2m1(VrT4) + sum_b l_ib v_mean[b]) / sum_b l_ib
 *   lse_i = ln 2 * (n + phi - 4 + log2 sum_b l_ib)   (optional)
 * PV runs as tcgen05 kind::mxf4nvf4 block-scaled MMAs.  Errors as
 * vca_attention_fwd; VCA_ERR_INVALID if v_sc is not 8-byte aligned. */
int vca_attention_fwd_fp4(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                          const float* k_scale, const uint8_t* VrT4, const uint8_t* v_sc,
                          const float* v_gscale, const vca_bf16* v_mean, int B, int H, int N, int d,
                          float softmax_scale, vca_bf16* O, float* lse, void* ws, size_t ws_bytes,
                          vca_stream_t stream);

/* Check of the block-scaled FP4 MMA that vca_attention_fwd_fp4 runs: one
 * 128x128x128 product in one CTA with known operands.  The pages have no
 * counterpart (a library self-test of the operand and scale-factor layouts).
 * All device pointers, 16-byte aligned:
 *   a_codes [128][64] bytes   A rows, E2M1 codes, low nibble = even column
 *   sf_cols [128][64] bytes   tensor-memory lane l, columns 0..15 (4 bytes
 *                             each): the A scale factors of K step k (64
 *                             columns of A) from column 4k, B's from 8 + 4k
 *   b_codes [128][64] bytes   B^T rows (one per output column), as a_codes
 *   D       [128][128] fp32   out: the product with the scales applied
 *   ws      status word (a wait that runs out records VCA_ERR_TIMEOUT) */
int vca_debug_fp4_mma(const uint8_t* a_codes, const uint8_t* sf_cols, const uint8_t* b_codes, float* D,
                      void* ws, vca_stream_t stream);

/* Same attention with Skip Softmax (BLASST) block rejection ([TRT-blog],
 * section "Sparse Attention with Skip Softmax": a score block is dropped for a
 * query row when exp(block max - running max) < lambda; dropped blocks skip the
 * exponentiation and their PV accumulation).  Row i drops key block b when
 *   z~_ib - max_{b' <= b} z~_ib' < log2(skip_lambda),  z~_ib = max_{j in b} z_ij
 * (z as in vca_attention_fwd, log2 units), except block 0, which is always
 * kept.  A dropped block adds no probabilities, no PV and a zero row sum; it
 * never moves the reference n.  When every row of a 128-row query tile drops a
 * block, the kernel also skips that tile's code pass and PV MMA.
 *   skip_lambda     in [0, 1); 0 gives exactly vca_attention_fwd
 *   skipped_tiles   optional device counter (one uint64, not zeroed here): the
 *                   number of (query tile, key block) pairs skipped is added
 * Errors as vca_attention_fwd, plus VCA_ERR_INVALID for skip_lambda outside
 * [0, 1). */
int vca_attention_fwd_skip(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                           const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                           const vca_bf16* v_mean, int B, int H, int N, int d, float softmax_scale,
                           float skip_lambda, vca_bf16* O, float* lse,
                           unsigned long long* skipped_tiles, void* ws, size_t ws_bytes,
                           vca_stream_t stream);

/* The whole path from host buffers to host buffers (grouping with
 * vca_cluster_permute from its default initialisation, vca_smooth_quantize_qkv,
 * vca_attention_fwd), with the copies overlapped with the kernels.  The pages
 * have no counterpart: it serves callers whose activations live in host memory.
 * (b, h) units are independent, so the layer runs in chunks of
 * up to `heads_per_chunk` units (0 = a quarter of the layer) through a
 * three-stage pipeline on library-owned streams over two device slots: copy
 * chunk c+1 in, compute chunk c, copy chunk c-1 out.  A slot takes its next
 * inputs as soon as the quantiser has read the previous ones, and its next
 * output once the previous one has been copied out.  Chunk sizes grow by 1.5x
 * from one unit up to heads_per_chunk and the last two chunks hold 3 units and
 * 1, so the transfers nothing overlaps stay small.  Results equal the three
 * calls on the whole layer bit for bit.
 *   Q, K, V   [B][H][N][d] bf16, HOST memory (in); page-locked memory
 *             (cudaHostAlloc / cudaHostRegister) is needed for the copies to
 *             overlap -- pageable memory works but serialises them
 *   O         [B][H][N][d] bf16, HOST memory (out)
 *   dev_buf   device scratch of vca_vc_attention_host_buffer_size() bytes,
 *             owned by the caller; its contents need no initialisation
 *   stream    the pipeline starts after the work queued on `stream`
 * Blocking: returns once O is written, with the first error of the host
 * checks, the launches or the device status words (bounded waits, non-finite
 * input).  d must be 128; 1 <= k <= VCA_MAX_CLUSTERS; iters >= 1. */
size_t vca_vc_attention_host_buffer_size(int B, int H, int N, int d, int k, int heads_per_chunk);
int vca_vc_attention_host(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H, int N,
                          int d, int k, int iters, float softmax_scale, vca_bf16* O, int heads_per_chunk,
                          void* dev_buf, size_t dev_bytes, vca_stream_t stream);

/* SAGE-style comparison recipe on the same harness ([TRT-blog], section
 * "Quantized Attention": q_block_size 1, k_block_size 16, v_block_size 1, FP8 V,
 * following the SageAttention2 line of work, whose K smoothing is applied).
 * Per (b, h), no reordering and no block means:
 *   k_mean[c]   = bf16(exact mean of K[:, c] over the N tokens)
 *   Qq, q_scale one fp32 scale per token: max|x| / 448, codes e4m3(x * 448/max|x|)
 *   Kq, k_scale K' = K - k_mean (fp32), one scale per 16 tokens, same formula
 *   VcT, v_chscale  one scale per channel over all N tokens, same formula;
 *               VcT is channel-major like VrT
 * An all-zero group has scale 1 and codes 0; padding rows and keys are 0.
 * Shapes: Qq, Kq [B][H][Np][d] u8; q_scale [B][H][Np] f32; k_scale
 * [B][H][Np/16] f32; VcT [B][H][d][Np] u8; v_chscale [B][H][d] f32; k_mean
 * [B][H][d] bf16.  |K| < 2^20 (exact fixed-point mean), finite inputs. */
size_t vca_sage_quantize_workspace_size(int B, int H, int N);
int vca_sage_quantize_qkv(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H, int N, int d,
                          uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale, uint8_t* VcT,
                          float* v_chscale, vca_bf16* k_mean, void* ws, size_t ws_bytes, vca_stream_t stream);

/* The FP8 attention of vca_attention_fwd (ExpCast codes, online reference,
 * tcgen05 MMAs) on SAGE-style operands: z uses the token's Q scale and the
 * 16-key group's K scale; PV has no block exponent and there is no mean
 * restore; output channel c is multiplied by v_chscale[c] after the
 * normalisation.  Workspace as vca_attention_fwd. */
int vca_attention_fwd_sage(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq, const float* k_scale,
                           const uint8_t* VcT, const float* v_chscale, int B, int H, int N, int d,
                           float softmax_scale, vca_bf16* O, float* lse, void* ws, size_t ws_bytes,
                           vca_stream_t stream);

/* The post's other qk_dtype, INT8 (the one it runs), on the same recipe:
 *   Qq, Kq int8 [B][H][Np][d]; q_scale = max|x| / 127 per token, k_scale the
 *   same per 16 smoothed keys; codes rne(x * (127 / max|x|)) with the product
 *   in fp32, in [-127, 127]; an all-zero group has scale 1 and codes 0.
 * V (E4M3, per channel), k_mean, padding, workspace and errors exactly as
 * vca_sage_quantize_qkv. */
int vca_sage_quantize_qkv_i8(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H, int N, int d,
                             int8_t* Qq, float* q_scale, int8_t* Kq, float* k_scale, uint8_t* VcT,
                             float* v_chscale, vca_bf16* k_mean, void* ws, size_t ws_bytes, vca_stream_t stream);

/* vca_attention_fwd_sage on the INT8 operands of vca_sage_quantize_qkv_i8:
 * QK^T is a tcgen05 kind::i8 MMA with s32 accumulation (exact: |q.k| < 2^21),
 * converted exactly to fp32 before z = s * q_scale * k_scale * softmax_scale *
 * log2(e); everything after that as vca_attention_fwd_sage. */
int vca_attention_fwd_sage_i8(const int8_t* Qq, const float* q_scale, const int8_t* Kq, const float* k_scale,
                              const uint8_t* VcT, const float* v_chscale, int B, int H, int N, int d,
                              float softmax_scale, vca_bf16* O, float* lse, void* ws, size_t ws_bytes,
                              vca_stream_t stream);

/* In-repo BF16 comparator: exact-softmax flash attention (online softmax with
 * exp2), tcgen05 BF16 MMAs with fp32 accumulation in tensor memory.
 *   Q, K, V, O [B][H][N][d] bf16; lse [B][H][N] fp32 natural log (nullable). */
size_t vca_bf16_attention_workspace_size(int B, int H, int N);
int vca_bf16_attention_fwd(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H,
                           int N, int d, float softmax_scale, vca_bf16* O, float* lse, void* ws,
                           size_t ws_bytes, vca_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* VCA_H */
