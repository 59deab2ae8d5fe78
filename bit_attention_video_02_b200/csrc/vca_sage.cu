// vca_sage.cu -- SAGE-style quantisation, the comparison recipe on the same
// harness ("Accelerating Video Generation with GEMM Quantization, Attention
// Quantization and Skip Softmax Attention in TensorRT-LLM", section "Quantized
// Attention": q_block_size 1, k_block_size 16, v_block_size 1, FP8 V; the
// SageAttention2 line of work it follows smooths K by its channel mean).
//
//   k_mean[c]   bf16 of the exact mean of K[:, c] over the head's N tokens
//   Q           one fp32 scale per token:        amax/448, e4m3(x * 448/amax)
//   K' = K - k_mean (fp32), one scale per 16 tokens, same formula
//   V           one scale per channel over all N tokens, same formula,
//               stored channel-major (VcT [d][Np]) like V-Smooth's residual
// No reordering and no block means: this is the recipe V-Smooth is compared to.
//
// qk_dtype int8 (the post's other choice, and the one it runs): Q and K' as
// signed bytes, amax/127 and rne(x * 127/amax), same groups; V stays E4M3.
//
// Three launches: channel statistics (exact K sums, V maxima), a tiny finalise
// (k_mean, per-channel V scales), and the quantisation of 128-token blocks.
#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

constexpr int kSageThreads = 256;
constexpr int kStatTok = 1024;   // tokens per statistics CTA: two runs of 512 per channel

struct SageWs {
  DevStatus* st;
  long long* ksum;   // [BH][128] exact fixed-point sums of K
  unsigned* vmax;    // [BH][128] max |V| as fp32 bits (non-negative floats order as integers)
  float* vinv;       // [BH][128] 448 / max |V| (0 for an all-zero channel)
};

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

static SageWs sage_carve(void* ws, int BH, size_t* total) {
  char* b = (char*)ws;
  size_t off = 0;
  SageWs w;
  w.st = (DevStatus*)(b + off);
  off += 256;
  w.ksum = (long long*)(b + off);
  off += al256((size_t)BH * 128 * sizeof(long long));
  w.vmax = (unsigned*)(b + off);
  off += al256((size_t)BH * 128 * sizeof(unsigned));
  w.vinv = (float*)(b + off);
  off += al256((size_t)BH * 128 * sizeof(float));
  *total = off;
  return w;
}

// Thread = (channel, half of the CTA's tokens).  A run of at most 512 tokens
// keeps each 22-bit half sum below 2^31.
__global__ void __launch_bounds__(kSageThreads) sage_stats_kernel(const uint16_t* __restrict__ K,
                                                                  const uint16_t* __restrict__ V,
                                                                  long long* __restrict__ ksum,
                                                                  unsigned* __restrict__ vmax, int N) {
  const int bh = blockIdx.y, ch = threadIdx.x & 127, half = threadIdx.x >> 7;
  const int n0 = blockIdx.x * kStatTok + half * (kStatTok / 2), n1 = min(N, n0 + kStatTok / 2);
  const uint16_t* kb = K + (int64_t)bh * N * 128 + ch;
  const uint16_t* vb = V + (int64_t)bh * N * 128 + ch;
  int hi = 0, lo = 0;
  float m = 0.0f;
#pragma unroll 8
  for (int n = n0; n < n1; ++n) {
    int h, l;
    fix24_split(__uint_as_float((uint32_t)__ldg(kb + (int64_t)n * 128) << 16), h, l);
    hi += h;
    lo += l;
    m = fmaxf(m, fabsf(__uint_as_float((uint32_t)__ldg(vb + (int64_t)n * 128) << 16)));
  }
  const long long s = ((long long)hi << 22) + (long long)lo;
  if (s != 0) atomicAdd(reinterpret_cast<unsigned long long*>(ksum + bh * 128 + ch), (unsigned long long)s);
  if (n0 < n1) atomicMax(vmax + bh * 128 + ch, __float_as_uint(m));
}

__global__ void sage_finalize_kernel(const long long* __restrict__ ksum, const unsigned* __restrict__ vmax,
                                     uint16_t* __restrict__ k_mean, float* __restrict__ v_chscale,
                                     float* __restrict__ vinv, int N) {
  const int i = blockIdx.x * 128 + threadIdx.x;
  k_mean[i] = double_to_bf16_rne(__ddiv_rn((double)ksum[i], (double)N * 16777216.0));
  const float m = __uint_as_float(vmax[i]);
  v_chscale[i] = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
  vinv[i] = m > 0.0f ? __fdiv_rn(448.0f, m) : 0.0f;
}

constexpr int kSageCodePitch = 144;   // bytes per shared row of the transposed V code tile

struct SageArgs {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const uint16_t* k_mean;
  const float* vinv;
  int N, nb;
  uint8_t* Qq;
  float* q_scale;    // [BH][Np]
  uint8_t* Kq;
  float* k_scale;    // [BH][Np/16]
  uint8_t* VcT;      // [BH][128][Np]
  int qk_i8;         // Q and K' as INT8 (amax/127, rne) instead of E4M3 (amax/448)
};

// Four fp32 values (already multiplied by 127/amax) as signed bytes, round to
// nearest even, in [-127, 127].
__device__ __forceinline__ uint32_t cvt_s8x4(float a, float b, float c, float d) {
  const int v[4] = {__float2int_rn(a), __float2int_rn(b), __float2int_rn(c), __float2int_rn(d)};
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) w |= (uint32_t)(min(127, max(-127, v[i])) & 0xFF) << (8 * i);
  return w;
}

// Eight codes of one thread's channels: x * inv rounded once in fp32, then
// coded as E4M3 (cvt, RNE, saturating) or as signed bytes.
__device__ __forceinline__ void c2_codes(const float (&x)[8], float inv, int qk_i8, uint32_t (&c2)[2]) {
  float y[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) y[c] = __fmul_rn(x[c], inv);
  if (qk_i8) {
    c2[0] = cvt_s8x4(y[0], y[1], y[2], y[3]);
    c2[1] = cvt_s8x4(y[4], y[5], y[6], y[7]);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) c2[q >> 1] |= (uint32_t)cvt_e4m3x2(y[2 * q], y[2 * q + 1]) << ((q & 1) * 16);
  }
}

// One CTA per (128-token block, tensor, head).  Thread t holds the 8 channels
// 8*(t%16).. of token rows 16*it + t/16 (it = 0..7), as 16-byte loads; the 16
// threads of a row sit in one half-warp, and the 16 rows of an `it` form one
// K scale group.
__global__ void __launch_bounds__(kSageThreads) sage_quant_kernel(const SageArgs a) {
  __shared__ __align__(16) uint8_t codeT[128 * kSageCodePitch];
  __shared__ float red[kSageThreads / 32][8];
  const int blk = blockIdx.x, tensor = blockIdx.y, bh = blockIdx.z;
  const int N = a.N;
  const int64_t Np = (int64_t)a.nb * 128;
  const int n0 = blk * 128, nv = min(128, N - n0);
  const int t = threadIdx.x, chunk = t & 15, rsub = t >> 4, lane = t & 31, warp = t >> 5;
  const uint16_t* src = (tensor == 0 ? a.Q : tensor == 1 ? a.K : a.V) + (int64_t)bh * N * 128;
  float x[8][8];   // [it][channel]
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int row = it * 16 + rsub;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (row < nv) w = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)(n0 + row) * 128) + chunk);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      x[it][2 * q] = bf16_lo(ws[q]);
      x[it][2 * q + 1] = bf16_hi(ws[q]);
    }
  }
  if (tensor == 0) {
    // ---- Q: one scale per token (the row's 16 threads share a half-warp)
    uint8_t* dst = a.Qq + ((int64_t)bh * Np + n0) * 128;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int row = it * 16 + rsub;
      float m = 0.0f;
#pragma unroll
      for (int c = 0; c < 8; ++c) m = fmaxf(m, fabsf(x[it][c]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const bool live = row < nv && m > 0.0f;
      const float qmax = a.qk_i8 ? 127.0f : 448.0f;
      const float inv = live ? __fdiv_rn(qmax, m) : 0.0f;
      uint32_t c2[2] = {0u, 0u};
      if (live) c2_codes(x[it], inv, a.qk_i8, c2);
      *reinterpret_cast<uint2*>(dst + (int64_t)row * 128 + chunk * 8) = make_uint2(c2[0], c2[1]);
      if (chunk == 0) a.q_scale[(int64_t)bh * Np + n0 + row] = live ? __fdiv_rn(m, qmax) : 1.0f;
    }
    return;
  }
  if (tensor == 1) {
    // ---- K: subtract the channel mean, then one scale per 16 tokens
    float mean[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) mean[c] = __uint_as_float((uint32_t)a.k_mean[bh * 128 + chunk * 8 + c] << 16);
    float gm[8];
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const bool row_ok = it * 16 + rsub < nv;
      float m = 0.0f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        x[it][c] = row_ok ? __fsub_rn(x[it][c], mean[c]) : 0.0f;
        m = fmaxf(m, fabsf(x[it][c]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      gm[it] = m;
    }
    if (lane == 0) {
#pragma unroll
      for (int it = 0; it < 8; ++it) red[warp][it] = gm[it];
    }
    __syncthreads();
    uint8_t* dst = a.Kq + ((int64_t)bh * Np + n0) * 128;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      float m = red[0][it];
#pragma unroll
      for (int w = 1; w < kSageThreads / 32; ++w) m = fmaxf(m, red[w][it]);
      const float qmax = a.qk_i8 ? 127.0f : 448.0f;
      const float inv = m > 0.0f ? __fdiv_rn(qmax, m) : 0.0f;
      const int row = it * 16 + rsub;
      uint32_t c2[2] = {0u, 0u};
      c2_codes(x[it], inv, a.qk_i8, c2);
      *reinterpret_cast<uint2*>(dst + (int64_t)row * 128 + chunk * 8) = make_uint2(c2[0], c2[1]);
      if (t == 0) a.k_scale[(int64_t)bh * (Np / 16) + blk * 8 + it] = m > 0.0f ? __fdiv_rn(m, qmax) : 1.0f;
    }
    return;
  }
  // ---- V: one scale per channel, codes transposed through shared memory
  float inv[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) inv[c] = a.vinv[bh * 128 + chunk * 8 + c];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int row = it * 16 + rsub;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t p = row < nv ? (uint32_t)cvt_e4m3x2(__fmul_rn(x[it][2 * q], inv[2 * q]),
                                                         __fmul_rn(x[it][2 * q + 1], inv[2 * q + 1]))
                                  : 0u;
      codeT[(chunk * 8 + 2 * q) * kSageCodePitch + row] = (uint8_t)(p & 0xFFu);
      codeT[(chunk * 8 + 2 * q + 1) * kSageCodePitch + row] = (uint8_t)(p >> 8);
    }
  }
  __syncthreads();
  uint8_t* dstT = a.VcT + (int64_t)bh * 128 * Np + n0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = i * kSageThreads + t;   // 0..1023: channel idx/8, 16-byte part idx%8
    const int c = idx >> 3, part = idx & 7;
    *reinterpret_cast<uint4*>(dstT + (int64_t)c * Np + part * 16) =
        *reinterpret_cast<const uint4*>(codeT + c * kSageCodePitch + part * 16);
  }
}

}  // namespace vca

using namespace vca;

extern "C" size_t vca_sage_quantize_workspace_size(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  size_t total;
  sage_carve(nullptr, B * H, &total);
  return total;
}

static int sage_quantize(const char* fn, const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H,
                         int N, int d, void* Qq, float* q_scale, void* Kq, float* k_scale, uint8_t* VcT,
                         float* v_chscale, vca_bf16* k_mean, void* ws, size_t ws_bytes, int qk_i8,
                         vca_stream_t stream) {
  if (d != VCA_HEAD_DIM) return fail(VCA_ERR_UNSUPPORTED, "%s: d must be 128", fn);
  if (B < 1 || H < 1 || N < 1 || (int64_t)B * H > 65535 || N > (1 << 24))
    return fail(VCA_ERR_INVALID, "%s: bad shape B=%d H=%d N=%d", fn, B, H, N);
  const void* ptrs[] = {Q, K, V, Qq, q_scale, Kq, k_scale, VcT, v_chscale, k_mean};
  for (const void* p : ptrs)
    if (!p) return fail(VCA_ERR_INVALID, "%s: null pointer", fn);
  const void* al16[] = {Q, K, V, Qq, Kq, VcT};
  for (const void* p : al16)
    if (!aligned16(p)) return fail(VCA_ERR_INVALID, "%s: tensors must be 16-byte aligned", fn);
  const int BH = B * H;
  if (!ws || ws_bytes < vca_sage_quantize_workspace_size(B, H, N))
    return fail(VCA_ERR_WORKSPACE, "%s: workspace too small", fn);
  size_t total;
  SageWs w = sage_carve(ws, BH, &total);
  cudaStream_t s = (cudaStream_t)stream;
  // the sums and maxima start at zero; the status word in front is left alone
  if (cudaMemsetAsync(w.ksum, 0, total - 256, s) != cudaSuccess) return fail(VCA_ERR_CUDA, "%s: memset failed", fn);
  sage_stats_kernel<<<dim3((N + kStatTok - 1) / kStatTok, BH), kSageThreads, 0, s>>>(K, V, w.ksum, w.vmax, N);
  int rc = check_launch("sage_stats_kernel");
  if (rc) return rc;
  sage_finalize_kernel<<<BH, 128, 0, s>>>(w.ksum, w.vmax, k_mean, v_chscale, w.vinv, N);
  if ((rc = check_launch("sage_finalize_kernel"))) return rc;
  SageArgs a;
  a.Q = Q; a.K = K; a.V = V; a.k_mean = k_mean; a.vinv = w.vinv; a.N = N; a.nb = (N + 127) / 128;
  a.Qq = (uint8_t*)Qq; a.q_scale = q_scale; a.Kq = (uint8_t*)Kq; a.k_scale = k_scale; a.VcT = VcT;
  a.qk_i8 = qk_i8;
  sage_quant_kernel<<<dim3(a.nb, 3, BH), kSageThreads, 0, s>>>(a);
  return check_launch("sage_quant_kernel");
}

extern "C" int vca_sage_quantize_qkv(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H,
                                     int N, int d, uint8_t* Qq, float* q_scale, uint8_t* Kq, float* k_scale,
                                     uint8_t* VcT, float* v_chscale, vca_bf16* k_mean, void* ws,
                                     size_t ws_bytes, vca_stream_t stream) {
  return sage_quantize("vca_sage_quantize_qkv", Q, K, V, B, H, N, d, Qq, q_scale, Kq, k_scale, VcT, v_chscale,
                       k_mean, ws, ws_bytes, 0, stream);
}

extern "C" int vca_sage_quantize_qkv_i8(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H,
                                        int N, int d, int8_t* Qq, float* q_scale, int8_t* Kq, float* k_scale,
                                        uint8_t* VcT, float* v_chscale, vca_bf16* k_mean, void* ws,
                                        size_t ws_bytes, vca_stream_t stream) {
  return sage_quantize("vca_sage_quantize_qkv_i8", Q, K, V, B, H, N, d, Qq, q_scale, Kq, k_scale, VcT, v_chscale,
                       k_mean, ws, ws_bytes, 1, stream);
}
