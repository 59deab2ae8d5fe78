// vca_prep.cu -- V-Smooth quantisation of Q, K and V (one fused launch).
//
// Method: "VC-Attention: Training-Free Low-Bit Attention Speeds Video Diffusion
// Up to 3.6x" (V-Smooth bullet): value tokens are reordered so each hardware
// block holds similar tokens, the block mean is subtracted and only the
// residual is quantised; "VC-Attention" (aikraft.ru, section "Решение"): the
// mean is stored exactly; "Nunchux AI Introduces VC-Attention..." (abstract):
// a mean costs 0.125 bit per value element (16 bits per 128 tokens).
//
// One CTA per (128-token block, tensor, head): 256 threads, HBM-bound; Q/K and
// V blocks are two launches of the same kernel (only V uses shared memory).  Loads
// are 16-byte vectors of whole token rows (gathered through the permutation for
// K and V); Q/K codes are written straight from registers, the V residual is
// transposed through shared memory so VrT rows (channel-major) are written as
// full 128-byte lines.
#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

constexpr int kPrepThreads = 256;
constexpr int kTilePitch = 136;            // bf16 elements per smem row (pad 8)
constexpr int kCodePitch = 144;            // bytes per smem row of the code tile

struct PrepArgs {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* perm;
  int N, nb;
  uint8_t* Qq;
  float* q_scale;
  uint8_t* Kq;
  float* k_scale;
  uint8_t* VrT;
  int8_t* v_exp;
  uint16_t* v_mean;
  DevStatus* st;
  int tensor_base;   // blockIdx.y + tensor_base: 0 = Q, 1 = K, 2 = V
};

// Smallest e with amax <= 448 * 2^e (0 for amax == 0), clamped to [-127, 127].
// amax = (1 + f) 2^(E-127) = ((1+f)/2) 2^(E-126); 448 = 0.875 2^9.
__device__ __forceinline__ int v_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  uint32_t u = __float_as_uint(amax);
  int E = (int)(u >> 23);
  if (E == 0) return -127;
  uint32_t f = u & 0x7FFFFFu;
  int e = (E - 126) - ((f <= 0x600000u) ? 9 : 8);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as an fp32 for e in [-127, 127] (2^127 down to 2^-127, the last subnormal).
__device__ __forceinline__ float pow2_neg(int e) {
  int k = -e;
  if (k >= -126) return __uint_as_float((uint32_t)(k + 127) << 23);
  return __uint_as_float(0x00400000u);  // 2^-127
}

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float m = red[0];
  for (int i = 1; i < kPrepThreads / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

__global__ void __launch_bounds__(kPrepThreads) smooth_quant_kernel(const PrepArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t* tile = reinterpret_cast<uint16_t*>(sm);                         // [128][136] bf16
  uint8_t* codeT = sm + 128 * kTilePitch * 2;                               // [128][144] u8
  __shared__ float red[kPrepThreads / 32];
  __shared__ long long psum[kPrepThreads];
  __shared__ float mu_s[128];
  __shared__ int flag_s;

  const int blk = blockIdx.x, tensor = blockIdx.y + a.tensor_base, bh = blockIdx.z;
  const int N = a.N, nb = a.nb;
  const int64_t Np = (int64_t)nb * 128;
  const int n0 = blk * 128;
  const int nv = min(128, N - n0);
  const int t = threadIdx.x;
  const int chunk = t & 15;          // 16-byte chunk (8 channels) of a row
  const int rsub = t >> 4;           // 0..15

  const uint16_t* src = tensor == 0 ? a.Q : (tensor == 1 ? a.K : a.V);
  src += (int64_t)bh * N * 128;
  const int32_t* perm = a.perm + (int64_t)bh * N;
  if (t == 0) flag_s = 0;
  __syncthreads();

  // ---- load 128 rows x 128 channels (8 rows of 16 per thread pass)
  uint4 w[8];
  float amax = 0.0f;
  int bad = 0;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    int row = it * 16 + rsub;
    w[it] = make_uint4(0, 0, 0, 0);
    if (row < nv) {
      int64_t srow = tensor == 0 ? (int64_t)(n0 + row) : (int64_t)__ldg(perm + n0 + row);
      w[it] = __ldg(reinterpret_cast<const uint4*>(src + srow * 128) + chunk);
      uint32_t ws4[4] = {w[it].x, w[it].y, w[it].z, w[it].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float lo = bf16_lo(ws4[q]), hi = bf16_hi(ws4[q]);
        amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
        uint32_t elo = (ws4[q] >> 7) & 0xFFu, ehi = (ws4[q] >> 23) & 0xFFu;
        bad |= (elo == 0xFF) | (ehi == 0xFF);
        if (tensor == 2) bad |= (elo >= 147) | (ehi >= 147);   // |v| >= 2^20
      }
    }
  }
  if (bad) flag_s = 1;

  if (tensor < 2) {
    // ---- Q / K: per-block fp32 scale, codes straight from registers
    float m = block_max(amax, red);
    if (flag_s && t == 0) report(a.st, VCA_ERR_NONFINITE, 1 + tensor, blk);
    float inv = 0.0f;
    if (m > 0.0f) inv = __fdiv_rn(448.0f, m);
    if (t == 0) {
      float* sc = tensor == 0 ? a.q_scale : a.k_scale;
      sc[(int64_t)bh * nb + blk] = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
    }
    uint8_t* dst = (tensor == 0 ? a.Qq : a.Kq) + ((int64_t)bh * Np + n0) * 128;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      int row = it * 16 + rsub;
      uint32_t ws4[4] = {w[it].x, w[it].y, w[it].z, w[it].w};
      uint32_t c[2] = {0u, 0u};
      if (row < nv && m > 0.0f) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t p = cvt_e4m3x2(__fmul_rn(bf16_lo(ws4[q]), inv), __fmul_rn(bf16_hi(ws4[q]), inv));
          c[q >> 1] |= p << ((q & 1) * 16);
        }
      }
      *reinterpret_cast<uint2*>(dst + (int64_t)row * 128 + chunk * 8) = make_uint2(c[0], c[1]);
    }
    return;
  }

  // ---- V: stage the block in shared memory
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    int row = it * 16 + rsub;
    *reinterpret_cast<uint4*>(tile + row * kTilePitch + chunk * 8) = w[it];
  }
  __syncthreads();
  if (flag_s && t == 0) report(a.st, VCA_ERR_NONFINITE, 3, blk);

  // exact per-channel sums in 2^-24 fixed point: two threads per channel
  const int ch = t & 127, half = t >> 7;
  long long s = 0;
  for (int r = half * 64; r < min(nv, half * 64 + 64); ++r) {
    float v = __uint_as_float((uint32_t)tile[r * kTilePitch + ch] << 16);
    s += __float2ll_rn(v * 16777216.0f);
  }
  psum[t] = s;
  __syncthreads();
  if (t < 128) {
    long long S = psum[t] + psum[t + 128];
    double mean = __ddiv_rn((double)S, (double)nv * 16777216.0);
    uint16_t mb = double_to_bf16_rne(mean);
    a.v_mean[((int64_t)bh * nb + blk) * 128 + t] = mb;
    mu_s[t] = __uint_as_float((uint32_t)mb << 16);
  }
  __syncthreads();

  // residual max over the valid tokens and all channels
  float mu = mu_s[ch];
  float ramax = 0.0f;
  for (int r = half * 64; r < min(nv, half * 64 + 64); ++r) {
    float v = __uint_as_float((uint32_t)tile[r * kTilePitch + ch] << 16);
    ramax = fmaxf(ramax, fabsf(__fsub_rn(v, mu)));
  }
  float m = block_max(ramax, red);
  int e = v_exponent(m);
  if (t == 0) a.v_exp[(int64_t)bh * nb + blk] = (int8_t)e;
  float sc = pow2_neg(e);

  // codes for (channel, 16 tokens) units -> transposed code tile
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int t0 = (half + 2 * i) * 16;
    uint32_t pk[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        int r = t0 + q * 4 + u;
        float v = __uint_as_float((uint32_t)tile[r * kTilePitch + ch] << 16);
        x[u] = r < nv ? __fmul_rn(__fsub_rn(v, mu), sc) : 0.0f;
      }
      pk[q] = (uint32_t)cvt_e4m3x2(x[0], x[1]) | ((uint32_t)cvt_e4m3x2(x[2], x[3]) << 16);
    }
    *reinterpret_cast<uint4*>(codeT + ch * kCodePitch + t0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  __syncthreads();
  // coalesced write: each VrT row (one channel) gets 128 bytes at tokens n0..n0+127
  uint8_t* dstT = a.VrT + (int64_t)bh * 128 * Np + n0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int idx = i * kPrepThreads + t;       // 0..1023
    int c = idx >> 3, part = idx & 7;
    *reinterpret_cast<uint4*>(dstT + (int64_t)c * Np + part * 16) =
        *reinterpret_cast<const uint4*>(codeT + c * kCodePitch + part * 16);
  }
}

constexpr size_t kPrepSmem = 128 * kTilePitch * 2 + 128 * kCodePitch;

// ---------------------------------------------------------------- 4-bit V-Smooth
// "Nunchux AI Introduces VC-Attention..." (abstract): a 4-bit V-Smooth serves
// workstation parts.  NVFP4 ("Accelerating Video Generation with GEMM
// Quantization, Attention Quantization and Skip Softmax Attention in
// TensorRT-LLM", table of quantisation formats): E2M1 elements, one E4M3 scale
// per 16 elements, one fp32 scale per tensor.  The V residual r = v - mean of a
// (b, h) head is coded in groups of 16 consecutive permuted tokens of one
// channel, with the head's tensor scale G = max|r| / (6 * 448):
//   group scale sc = e4m3(amax_g / (6 G)), codes e2m1(r * (1 / (decode(sc) G)))
// (each product, quotient and reciprocal rounded once in fp32).  Q, K and the
// block means are exactly those of the 8-bit prep.  Two passes over V: the
// first writes the block means and folds each block's residual maximum into
// its head's (atomic max on the fp32 bits, which order like unsigned integers
// for non-negative values); the second reloads the block, rebuilds the
// residual from the stored bf16 mean and codes it.  Layouts: VrT4 [d][Np/2]
// per head, token j of channel c in byte j/2 of row c, low nibble for even j;
// v_sc [d][Np/16] per head.

constexpr int kV4Pitch = 80;   // bytes per smem row of the 4-bit tile: 64 code bytes + 8 scales + pad

struct PrepV4Args {
  const uint16_t* V;
  const int32_t* perm;
  int N, nb;
  uint8_t* VrT4;
  uint8_t* v_sc;
  float* v_gscale;
  uint16_t* v_mean;
  unsigned* head_amax;   // [B*H] fp32 bits of max|r|, zeroed before the first pass
  DevStatus* st;
};

// Nearest E2M1 value (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6) to x, ties to the
// even code, finite values saturating at 6; the sign goes to bit 3.
__device__ __forceinline__ uint32_t e2m1_code(float x) {
  const float a = fabsf(x);
  const uint32_t c = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
                   : a <= 2.5f  ? 4u : a < 3.5f  ? 5u : a <= 5.0f  ? 6u : 7u;
  return c | ((__float_as_uint(x) >> 31) << 3);
}

template <int PASS>
__global__ void __launch_bounds__(kPrepThreads) smooth_quant_v4_kernel(const PrepV4Args a) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t* tile = reinterpret_cast<uint16_t*>(sm);     // [128][136] bf16
  uint8_t* codeT = sm + 128 * kTilePitch * 2;           // [128][80] u8 (second pass)
  __shared__ float red[kPrepThreads / 32];
  __shared__ long long psum[kPrepThreads];
  __shared__ float mu_s[128];
  __shared__ int flag_s;

  const int blk = blockIdx.x, bh = blockIdx.y;
  const int N = a.N, nb = a.nb;
  const int64_t Np = (int64_t)nb * 128;
  const int n0 = blk * 128;
  const int nv = min(128, N - n0);
  const int t = threadIdx.x;
  const int chunk = t & 15, rsub = t >> 4;
  const uint16_t* src = a.V + (int64_t)bh * N * 128;
  const int32_t* perm = a.perm + (int64_t)bh * N;
  if (t == 0) flag_s = 0;
  __syncthreads();

  // ---- gather the block's 128 permuted value rows into shared memory
  int bad = 0;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int row = it * 16 + rsub;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (row < nv) {
      w = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)__ldg(perm + n0 + row) * 128) + chunk);
      if (PASS == 0) {
        const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t elo = (ws4[q] >> 7) & 0xFFu, ehi = (ws4[q] >> 23) & 0xFFu;
          bad |= (elo >= 147) | (ehi >= 147);   // non-finite or |v| >= 2^20
        }
      }
    }
    *reinterpret_cast<uint4*>(tile + row * kTilePitch + chunk * 8) = w;
  }
  if (bad) flag_s = 1;
  __syncthreads();
  const int ch = t & 127, half = t >> 7;

  if (PASS == 0) {
    if (flag_s && t == 0) report(a.st, VCA_ERR_NONFINITE, 3, blk);
    // exact per-channel sums in 2^-24 fixed point (two threads per channel),
    // one fp64 division, one rounding to bf16: the 8-bit prep's block mean
    long long s = 0;
    for (int r = half * 64; r < min(nv, half * 64 + 64); ++r)
      s += __float2ll_rn(__uint_as_float((uint32_t)tile[r * kTilePitch + ch] << 16) * 16777216.0f);
    psum[t] = s;
    __syncthreads();
    if (t < 128) {
      const long long S = psum[t] + psum[t + 128];
      const uint16_t mb = double_to_bf16_rne(__ddiv_rn((double)S, (double)nv * 16777216.0));
      a.v_mean[((int64_t)bh * nb + blk) * 128 + t] = mb;
      mu_s[t] = __uint_as_float((uint32_t)mb << 16);
    }
    __syncthreads();
    const float mu = mu_s[ch];
    float ramax = 0.0f;
    for (int r = half * 64; r < min(nv, half * 64 + 64); ++r)
      ramax = fmaxf(ramax, fabsf(__fsub_rn(__uint_as_float((uint32_t)tile[r * kTilePitch + ch] << 16), mu)));
    const float m = block_max(ramax, red);
    if (t == 0) atomicMax(a.head_amax + bh, __float_as_uint(m));
    return;
  }

  // ---- second pass: code (channel, 16-token group) units, four per thread
  if (t < 128) mu_s[t] = __uint_as_float((uint32_t)a.v_mean[((int64_t)bh * nb + blk) * 128 + t] << 16);
  __syncthreads();
  const float hmax = __uint_as_float(a.head_amax[bh]);
  const float G = hmax > 0.0f ? __fdiv_rn(hmax, 2688.0f) : 1.0f;
  if (blk == 0 && t == 0) a.v_gscale[bh] = G;
  const float sixG = __fmul_rn(6.0f, G);
  const float mu = mu_s[ch];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int g = half + 2 * i;   // group of the block: tokens 16g .. 16g+15
    float x[16];
    float am = 0.0f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int r = g * 16 + u;
      const float v = __uint_as_float((uint32_t)tile[r * kTilePitch + ch] << 16);
      x[u] = r < nv ? __fsub_rn(v, mu) : 0.0f;
      am = fmaxf(am, fabsf(x[u]));
    }
    const uint32_t sc = cvt_e4m3x2(__fdiv_rn(am, sixG), 0.0f) & 0xFFu;
    const float sg = __fmul_rn(__uint_as_float(sc << 20) * 0x1p120f, G);   // decode(sc) * G
    uint32_t lo = 0u, hi = 0u;
    if (sg > 0.0f) {
      const float inv = __frcp_rn(sg);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        lo |= e2m1_code(__fmul_rn(x[u], inv)) << (4 * u);
        hi |= e2m1_code(__fmul_rn(x[u + 8], inv)) << (4 * u);
      }
    }
    *reinterpret_cast<uint2*>(codeT + ch * kV4Pitch + g * 8) = make_uint2(lo, hi);
    codeT[ch * kV4Pitch + 64 + g] = (uint8_t)sc;
  }
  __syncthreads();
  // coalesced writes: 64 code bytes per channel row of VrT4, 8 scale bytes per row of v_sc
  uint8_t* dst = a.VrT4 + (int64_t)bh * 128 * (Np / 2) + blk * 64;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int idx = i * kPrepThreads + t;   // 0..511
    const int c = idx >> 2, part = idx & 3;
    *reinterpret_cast<uint4*>(dst + (int64_t)c * (Np / 2) + part * 16) =
        *reinterpret_cast<const uint4*>(codeT + c * kV4Pitch + part * 16);
  }
  if (t < 128)
    *reinterpret_cast<uint2*>(a.v_sc + ((int64_t)bh * 128 + t) * (Np / 16) + blk * 8) =
        *reinterpret_cast<const uint2*>(codeT + t * kV4Pitch + 64);
}

constexpr size_t kV4Smem0 = 128 * kTilePitch * 2;
constexpr size_t kV4Smem1 = kV4Smem0 + 128 * kV4Pitch;

}  // namespace vca

using namespace vca;

extern "C" size_t vca_smooth_quantize_workspace_size(int B, int H, int N) {
  return 256;  // status word only
}

extern "C" int vca_smooth_quantize_qkv(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V,
                                       const int32_t* perm, int B, int H, int N, int d, int block,
                                       uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                                       uint8_t* VrT, int8_t* v_exp, vca_bf16* v_mean, void* ws,
                                       size_t ws_bytes, vca_stream_t stream) {
  if (d != VCA_HEAD_DIM) return fail(VCA_ERR_UNSUPPORTED, "vca_smooth_quantize_qkv: d must be 128");
  if (block != VCA_BLOCK) return fail(VCA_ERR_UNSUPPORTED, "vca_smooth_quantize_qkv: block must be 128");
  if (B < 1 || H < 1 || N < 1 || (int64_t)B * H > 65535 || N > (1 << 24))
    return fail(VCA_ERR_INVALID, "vca_smooth_quantize_qkv: bad shape B=%d H=%d N=%d", B, H, N);
  const void* ptrs[] = {Q, K, V, perm, Qq, q_scale, Kq, k_scale, VrT, v_exp, v_mean};
  for (const void* p : ptrs)
    if (!p) return fail(VCA_ERR_INVALID, "vca_smooth_quantize_qkv: null pointer");
  const void* al16[] = {Q, K, V, Qq, Kq, VrT};
  for (const void* p : al16)
    if (!aligned16(p)) return fail(VCA_ERR_INVALID, "vca_smooth_quantize_qkv: tensors must be 16-byte aligned");
  if (!ws || ws_bytes < vca_smooth_quantize_workspace_size(B, H, N))
    return fail(VCA_ERR_WORKSPACE, "vca_smooth_quantize_qkv: workspace too small");
  if (cudaFuncSetAttribute(smooth_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kPrepSmem) != cudaSuccess)
    return fail(VCA_ERR_CUDA, "vca_smooth_quantize_qkv: cannot set shared-memory size");
  PrepArgs a;
  a.Q = Q; a.K = K; a.V = V; a.perm = perm; a.N = N; a.nb = (N + 127) / 128;
  a.Qq = Qq; a.q_scale = q_scale; a.Kq = Kq; a.k_scale = k_scale; a.VrT = VrT;
  a.v_exp = v_exp; a.v_mean = v_mean; a.st = (DevStatus*)ws;
  // Q and K blocks need no shared tile: a launch of their own keeps them at full
  // occupancy; the V blocks (mean, residual, transpose) get the shared tile
  a.tensor_base = 0;
  smooth_quant_kernel<<<dim3(a.nb, 2, B * H), kPrepThreads, 0, (cudaStream_t)stream>>>(a);
  int rc = check_launch("smooth_quant_kernel (Q, K)");
  if (rc) return rc;
  a.tensor_base = 2;
  smooth_quant_kernel<<<dim3(a.nb, 1, B * H), kPrepThreads, kPrepSmem, (cudaStream_t)stream>>>(a);
  return check_launch("smooth_quant_kernel (V)");
}

extern "C" size_t vca_smooth_quantize_fp4_workspace_size(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  return 256 + (((size_t)B * H * 4 + 255) & ~(size_t)255);   // status word + one max per head
}

extern "C" int vca_smooth_quantize_qkv_fp4(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V,
                                           const int32_t* perm, int B, int H, int N, int d, uint8_t* Qq,
                                           float* q_scale, uint8_t* Kq, float* k_scale, uint8_t* VrT4,
                                           uint8_t* v_sc, float* v_gscale, vca_bf16* v_mean, void* ws,
                                           size_t ws_bytes, vca_stream_t stream) {
  const char* fn = "vca_smooth_quantize_qkv_fp4";
  if (d != VCA_HEAD_DIM) return fail(VCA_ERR_UNSUPPORTED, "%s: d must be 128", fn);
  if (B < 1 || H < 1 || N < 1 || (int64_t)B * H > 65535 || N > (1 << 24))
    return fail(VCA_ERR_INVALID, "%s: bad shape B=%d H=%d N=%d", fn, B, H, N);
  const void* ptrs[] = {Q, K, V, perm, Qq, q_scale, Kq, k_scale, VrT4, v_sc, v_gscale, v_mean};
  for (const void* p : ptrs)
    if (!p) return fail(VCA_ERR_INVALID, "%s: null pointer", fn);
  const void* al16[] = {Q, K, V, Qq, Kq, VrT4, v_sc};
  for (const void* p : al16)
    if (!aligned16(p)) return fail(VCA_ERR_INVALID, "%s: tensors must be 16-byte aligned", fn);
  if (!ws || ws_bytes < vca_smooth_quantize_fp4_workspace_size(B, H, N))
    return fail(VCA_ERR_WORKSPACE, "%s: workspace too small", fn);
  const int nb = (N + 127) / 128;
  cudaStream_t s = (cudaStream_t)stream;
  // Q and K: the 8-bit prep's kernel, unchanged
  PrepArgs a;
  a.Q = Q; a.K = K; a.V = V; a.perm = perm; a.N = N; a.nb = nb;
  a.Qq = Qq; a.q_scale = q_scale; a.Kq = Kq; a.k_scale = k_scale; a.VrT = nullptr;
  a.v_exp = nullptr; a.v_mean = nullptr; a.st = (DevStatus*)ws; a.tensor_base = 0;
  smooth_quant_kernel<<<dim3(nb, 2, B * H), kPrepThreads, 0, s>>>(a);
  int rc = check_launch("smooth_quant_kernel (Q, K)");
  if (rc) return rc;
  // V: block means and the head maxima, then the NVFP4 residual
  PrepV4Args v;
  v.V = V; v.perm = perm; v.N = N; v.nb = nb; v.VrT4 = VrT4; v.v_sc = v_sc; v.v_gscale = v_gscale;
  v.v_mean = v_mean; v.head_amax = reinterpret_cast<unsigned*>((char*)ws + 256); v.st = (DevStatus*)ws;
  if (cudaMemsetAsync(v.head_amax, 0, (size_t)B * H * 4, s) != cudaSuccess)
    return fail(VCA_ERR_CUDA, "%s: memset failed", fn);
  smooth_quant_v4_kernel<0><<<dim3(nb, B * H), kPrepThreads, kV4Smem0, s>>>(v);
  rc = check_launch("smooth_quant_v4_kernel<0>");
  if (rc) return rc;
  smooth_quant_v4_kernel<1><<<dim3(nb, B * H), kPrepThreads, kV4Smem1, s>>>(v);
  return check_launch("smooth_quant_v4_kernel<1>");
}
