// vca_prep.cu -- V-Smooth quantisation of Q, K and V.
//
// Method: "VC-Attention: Training-Free Low-Bit Attention Speeds Video Diffusion
// Up to 3.6x" (V-Smooth bullet): value tokens are reordered so each hardware
// block holds similar tokens, the block mean is subtracted and only the
// residual is quantised; "VC-Attention" (aikraft.ru, section "Решение"): the
// mean is stored exactly; "Nunchux AI Introduces VC-Attention..." (abstract):
// a mean costs 0.125 bit per value element (16 bits per 128 tokens).
//
// vca_smooth_quantize_qkv runs one persistent kernel (smooth_quant_stream_kernel):
// a producer warp streams 128-token tiles of Q, K and V (K and V rows gathered
// through the permutation) into a 3-stage shared-memory ring with 16-byte
// asynchronous copies, and 8 compute warps code one tile while two more land.
// Q/K tiles: per-block fp32 scale, codes written straight from registers.
// V tiles: each thread holds 8 consecutive tokens x 8 channels; exact
// per-channel sums and the residual maximum through shared-memory reductions;
// the residual codes are transposed in registers so VrT rows (channel-major)
// are written as full 128-byte lines.  The 4-bit prep runs the same kernel for
// Q, K and its first pass over V (block means, heads' residual maxima), then
// smooth_quant_v4_kernel codes the NVFP4 residual.
#include <algorithm>

#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

constexpr int kPrepThreads = 256;
constexpr int kTilePitch = 136;            // bf16 elements per smem row (pad 8)

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
  // 4-bit prep, first pass over V (streaming kernel): V blocks write their means
  // and fold their residual maximum into head_amax[bh] instead of being coded
  unsigned* head_amax;
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

// 4 x 4 byte transpose: out[c] byte r = in[r] byte c.
__device__ __forceinline__ void transpose4x4(const uint32_t in[4], uint32_t out[4]) {
  const uint32_t t0 = prmt(in[0], in[1], 0x5140u), t1 = prmt(in[0], in[1], 0x7362u);
  const uint32_t t2 = prmt(in[2], in[3], 0x5140u), t3 = prmt(in[2], in[3], 0x7362u);
  out[0] = prmt(t0, t2, 0x5410u);
  out[1] = prmt(t0, t2, 0x7632u);
  out[2] = prmt(t1, t3, 0x5410u);
  out[3] = prmt(t1, t3, 0x7632u);
}


// V code tile: 128 channel rows of 128 bytes; the 8-byte segment of tokens
// 8 g .. 8 g + 7 of channel c sits at segment g ^ (2 ((c >> 3) & 7)), so the 32
// threads of a warp storing one channel each hit 16 bank pairs twice, and
// 16-byte parts keep adjacent token segments together.
__device__ __forceinline__ int vseg_swz(int c) { return 2 * ((c >> 3) & 7); }

// ---------------------------------------------------------------- streaming form
// vca_smooth_quantize_qkv's kernel: persistent CTAs walk the (block, tensor,
// head) items; a producer warp (warp 8) fills a 3-stage ring of 32 KB token
// tiles with 16-byte asynchronous copies (cp.async; for K and V each
// instruction moves two whole gathered rows, lanes 0-15 and 16-31), so two
// blocks stream in while the 8 compute warps code one.  (One bulk copy per
// 256-byte gathered row kept the copy engine busy: the K and V tiles waited
// ~4,000 cycles for their rows against ~120 for a Q tile in one bulk copy.)  The compute warps synchronise
// among themselves on named barrier 1 and release a stage with one arrival
// per warp.  The V scratch (exact partial sums and the code tile) reuses the
// stage of the block being coded.
constexpr int kStreamStages = 3;
constexpr uint32_t kStageBytes = 128 * 256;
constexpr size_t kStreamSmem = kStreamStages * kStageBytes + 128;
constexpr int kStreamThreads = kPrepThreads + 32;

__device__ __forceinline__ void compute_sync() {   // the 256 compute threads
  asm volatile("bar.sync 1, %0;" ::"n"(kPrepThreads) : "memory");
}
__device__ __forceinline__ int compute_sync_or(int pred) {
  int r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\t"
               "selp.s32 %0, 1, 0, q;\n\t}"
               : "=r"(r)
               : "r"(pred), "n"(kPrepThreads)
               : "memory");
  return r;
}
// Maximum of v over the 256 compute threads, and the OR of pred, with one
// barrier.  red[] is rewritten here, so no thread may still be reading it
// from an earlier call: every call is separated from the previous one by a
// compute barrier (the per-item barrier at the top of the loop).
__device__ __forceinline__ float compute_max_or(float v, int pred, float* red, int& any) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  any = compute_sync_or(pred);
  float m = red[0];
  for (int i = 1; i < kPrepThreads / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

// 16 bytes global -> shared (cp.async, cached in L2 only); completion is
// reported through cp_async_mbar_arrive.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// Arrive on the barrier once every cp.async this thread issued before has
// completed (.noinc: the arrival is one of the barrier's expected count).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}


// Per 16-bit half, the larger of the two bf16 magnitude bit patterns (for
// finite values these order like the magnitudes; inf and NaN are larger).
__device__ __forceinline__ uint32_t vmax_mag2(uint32_t acc, uint32_t w) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w & 0x7FFF7FFFu));
  return r;
}
__device__ __forceinline__ uint32_t max_half(uint32_t m2) { return max(m2 & 0xFFFFu, m2 >> 16); }

__global__ void __launch_bounds__(kStreamThreads, 2) smooth_quant_stream_kernel(const PrepArgs a, int BH,
                                                                                 unsigned long long lim) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t full[kStreamStages];
  __shared__ uint64_t empty[kStreamStages];
  __shared__ float red[kPrepThreads / 32];
  __shared__ float mu_s[128];
  __shared__ int abort_s;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int N = a.N, nb = a.nb;
  const int64_t Np = (int64_t)nb * 128;
  if (t == 0) {
    abort_s = 0;
    for (int i = 0; i < kStreamStages; ++i) {
      mbar_init(&full[i], 32);   // one arrival per producer lane
      mbar_init(&empty[i], kPrepThreads / 32);
    }
    fence_barrier_init();
  }
  __syncthreads();
  // Items it = blockIdx.x + k * gridDim.x, it = 3 (bh nb + blk) + tensor
  // (tensors interleaved so a CTA mixes all three), walked by a cursor that
  // adds the stride with carries: no 64-bit division per item.
  struct Cursor {
    int tensor, blk, bh;
  };
  const int step = gridDim.x;
  const int st_t = step % 3, st_q = step / 3, st_b = st_q % nb, st_h = st_q / nb;
  auto first_item = [&]() {
    const int it = blockIdx.x, q = it / 3;
    return Cursor{it % 3, q % nb, q / nb};
  };
  auto next_item = [&](Cursor& c) {
    c.tensor += st_t;
    const int c1 = c.tensor >= 3;
    c.tensor -= 3 * c1;
    c.blk += st_b + c1;
    const int c2 = c.blk >= nb;
    c.blk -= nb * c2;
    c.bh += st_h + c2;
  };
  if (warp == kPrepThreads / 32) {
    // ---- producer: item k goes to stage k % 3 once the compute warps released it
    int k = 0;
    for (Cursor cur = first_item(); cur.bh < BH; next_item(cur), ++k) {
      const int stg = k % kStreamStages;
      if (k >= kStreamStages &&
          !mbar_wait_bounded(&empty[stg], ((k / kStreamStages) - 1) & 1, &abort_s, a.st, lim, 803))
        break;
      const int tensor = cur.tensor, bh = cur.bh, blk = cur.blk;
      const int n0 = blk * 128, nv = min(128, N - n0);
      uint8_t* dst = stages + stg * kStageBytes;
      if (tensor == 0) {
        // Q rows are contiguous: lane l copies 16-byte chunks l, l + 32, ...
        const uint8_t* src = reinterpret_cast<const uint8_t*>(a.Q + ((int64_t)bh * N + n0) * 128);
        for (int c = lane; c < nv * 16; c += 32) cp_async16(dst + c * 16, src + (int64_t)c * 16);
      } else {
        // gathered rows: the source indices first (one round trip), then per
        // instruction two whole 256-byte rows (lanes 0-15 and 16-31)
        const int32_t* pm = a.perm + (int64_t)bh * N + n0;
        int src_row[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) src_row[i] = lane + 32 * i < nv ? __ldg(pm + lane + 32 * i) : 0;
        const uint8_t* src = reinterpret_cast<const uint8_t*>((tensor == 1 ? a.K : a.V) + (int64_t)bh * N * 128);
        const int half = lane >> 4, ch = lane & 15;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int r = 32 * j + 2 * i + half;
            const int srow = __shfl_sync(0xffffffffu, src_row[j], 2 * i + half);
            if (r < nv) cp_async16(dst + r * 256 + ch * 16, src + (int64_t)srow * 256 + ch * 16);
          }
        }
      }
      // one arrival per lane, made once all of the lane's copies have landed
      cp_async_mbar_arrive(&full[stg]);
    }
    return;
  }
  int k = 0;
  for (Cursor cur = first_item(); cur.bh < BH; next_item(cur), ++k) {
    const int stg = k % kStreamStages;
    uint8_t* tile = stages + stg * kStageBytes;
    bool ok = mbar_wait_bounded(&full[stg], (k / kStreamStages) & 1, &abort_s, a.st, lim, 800);
    if (compute_sync_or(!ok)) break;
    const int tensor = cur.tensor, bh = cur.bh, blk = cur.blk;
    const int n0 = blk * 128, nv = min(128, N - n0);
    if (tensor < 2) {
      // ---- Q / K: per-block fp32 scale, codes straight from registers
      const int chunk = t & 15, rsub = t >> 4;
      uint4 w[8];
      uint32_t m2 = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = i * 16 + rsub;
        w[i] = row < nv ? *reinterpret_cast<const uint4*>(tile + row * 256 + chunk * 16) : make_uint4(0, 0, 0, 0);
        m2 = vmax_mag2(vmax_mag2(m2, w[i].x), w[i].y);
        m2 = vmax_mag2(vmax_mag2(m2, w[i].z), w[i].w);
      }
      const uint32_t mbits = max_half(m2);
      int nonfinite;
      const float m = compute_max_or(__uint_as_float(mbits << 16), mbits >= 0x7F80u, red, nonfinite);   // block max |x|
      if (nonfinite && t == 0) report(a.st, VCA_ERR_NONFINITE, 1 + tensor, blk);
      const float inv = m > 0.0f ? __fdiv_rn(448.0f, m) : 0.0f;
      if (t == 0) (tensor == 0 ? a.q_scale : a.k_scale)[(int64_t)bh * nb + blk] = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
      uint8_t* dst = (tensor == 0 ? a.Qq : a.Kq) + ((int64_t)bh * Np + n0) * 128;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = i * 16 + rsub;
        const uint32_t ws4[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
        uint32_t c[2] = {0u, 0u};
        if (row < nv && m > 0.0f) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 y = __fmul2_rn(make_float2(bf16_lo(ws4[q]), bf16_hi(ws4[q])), make_float2(inv, inv));
            c[q >> 1] |= (uint32_t)cvt_e4m3x2(y.x, y.y) << ((q & 1) * 16);
          }
        }
        *reinterpret_cast<uint2*>(dst + (int64_t)row * 128 + chunk * 8) = make_uint2(c[0], c[1]);
      }
    } else {
      // ---- V: thread = 8 consecutive tokens x 8 channels
      const int chunk = t & 15, g = t >> 4;
      uint4 w[8];
      uint32_t m2 = 0u;
      // exact fixed-point sums: llrint(v 2^24) = hi 2^22 + lo per value (the
      // split of fix24_split, two values per fma.rn.f32x2), summed as the raw
      // bits magic + hi and magic + lo; the 8 magic constants of the 8 tokens
      // are taken off once (wrap-around arithmetic, |sum| < 2^26)
      uint32_t hs[8], ls[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) hs[c] = ls[c] = 0u;
      const float kMagic = 12582912.0f;   // 1.5 * 2^23
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int row = 8 * g + u;
        w[u] = row < nv ? *reinterpret_cast<const uint4*>(tile + row * 256 + chunk * 16) : make_uint4(0, 0, 0, 0);
        m2 = vmax_mag2(vmax_mag2(m2, w[u].x), w[u].y);
        m2 = vmax_mag2(vmax_mag2(m2, w[u].z), w[u].w);
        const uint32_t ws4[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 v = make_float2(bf16_lo(ws4[q]), bf16_hi(ws4[q]));
          // hm = magic + rne(4 v); r = v - hi / 4 (exact); lm = magic + rne(r 2^24)
          const float2 hm = __ffma2_rn(v, make_float2(4.0f, 4.0f), make_float2(kMagic, kMagic));
          const float2 hf = __fadd2_rn(hm, make_float2(-kMagic, -kMagic));
          const float2 rr = __ffma2_rn(hf, make_float2(-0.25f, -0.25f), v);
          const float2 lm = __ffma2_rn(rr, make_float2(16777216.0f, 16777216.0f), make_float2(kMagic, kMagic));
          hs[2 * q] += __float_as_uint(hm.x);
          hs[2 * q + 1] += __float_as_uint(hm.y);
          ls[2 * q] += __float_as_uint(lm.x);
          ls[2 * q + 1] += __float_as_uint(lm.y);
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        hs[c] -= 8u * 0x4B400000u;
        ls[c] -= 8u * 0x4B400000u;
      }
      // the tile is in registers: its stage now holds the partial sums and codes
      const bool anybad = compute_sync_or(max_half(m2) >= 0x4980u);   // |v| >= 2^20, inf or NaN
      if (anybad && t == 0) report(a.st, VCA_ERR_NONFINITE, 3, blk);
      int* s_hi = reinterpret_cast<int*>(tile);
      int* s_lo = s_hi + 16 * 128;
      uint8_t* codeT = tile + 2 * 16 * 128 * 4;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        s_hi[g * 128 + 8 * chunk + c] = (int)hs[c];
        s_lo[g * 128 + 8 * chunk + c] = (int)ls[c];
      }
      compute_sync();
      if (t < 128) {
        int H = 0, L = 0;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          H += s_hi[q * 128 + t];
          L += s_lo[q * 128 + t];
        }
        const long long S = (long long)H * 4194304ll + (long long)L;
        // S / (nv 2^24): for a full block a division by 2^31, exact as a product
        const double mean = nv == 128 ? (double)S * 0x1p-31 : __ddiv_rn((double)S, (double)nv * 16777216.0);
        const uint16_t mb = double_to_bf16_rne(mean);
        a.v_mean[((int64_t)bh * nb + blk) * 128 + t] = mb;
        mu_s[t] = __uint_as_float((uint32_t)mb << 16);
      }
      compute_sync();
      float mu[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mu[c] = mu_s[8 * chunk + c];
      float ramax = 0.0f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (8 * g + u < nv) {
          const uint32_t ws4[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 y = __fadd2_rn(make_float2(bf16_lo(ws4[q]), bf16_hi(ws4[q])),
                                        make_float2(-mu[2 * q], -mu[2 * q + 1]));
            ramax = fmax3(ramax, fabsf(y.x), fabsf(y.y));
          }
        }
      }
      int unused;
      const float m = compute_max_or(ramax, 0, red, unused);
      if (a.head_amax) {
        // 4-bit prep, first pass: the head's residual maximum (fp32 bits of a
        // non-negative value order like unsigned integers); coding comes later
        if (t == 0) atomicMax(a.head_amax + bh, __float_as_uint(m));
      } else {
      const int e = v_exponent(m);
      if (t == 0) a.v_exp[(int64_t)bh * nb + blk] = (int8_t)e;
      const float sc = pow2_neg(e);
      float musc[8];   // -mu * 2^-e (exact: a power of two times a bf16 value)
#pragma unroll
      for (int c = 0; c < 8; ++c) musc[c] = -mu[c] * sc;
      uint32_t lo4[8], hi4[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t ws4[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        // (v - mu) * 2^-e, rounded once to fp32 by the subtraction; the power of
        // two is applied exactly inside the same fma (fp32 results below 2^-126
        // code to E4M3 zero either way)
        float x[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 y = __ffma2_rn(make_float2(bf16_lo(ws4[q]), bf16_hi(ws4[q])), make_float2(sc, sc),
                                      make_float2(musc[2 * q], musc[2 * q + 1]));
          x[2 * q] = y.x;
          x[2 * q + 1] = y.y;
        }
        const bool valid = 8 * g + u < nv;
        lo4[u] = valid ? ((uint32_t)cvt_e4m3x2(x[0], x[1]) | ((uint32_t)cvt_e4m3x2(x[2], x[3]) << 16)) : 0u;
        hi4[u] = valid ? ((uint32_t)cvt_e4m3x2(x[4], x[5]) | ((uint32_t)cvt_e4m3x2(x[6], x[7]) << 16)) : 0u;
      }
      uint32_t cT[8][2];
      {
        uint32_t o[4];
        transpose4x4(lo4, o);
        for (int c = 0; c < 4; ++c) cT[c][0] = o[c];
        transpose4x4(lo4 + 4, o);
        for (int c = 0; c < 4; ++c) cT[c][1] = o[c];
        transpose4x4(hi4, o);
        for (int c = 0; c < 4; ++c) cT[4 + c][0] = o[c];
        transpose4x4(hi4 + 4, o);
        for (int c = 0; c < 4; ++c) cT[4 + c][1] = o[c];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = 8 * chunk + i;
        *reinterpret_cast<uint2*>(codeT + c * 128 + 8 * (g ^ vseg_swz(c))) = make_uint2(cT[i][0], cT[i][1]);
      }
      compute_sync();
      uint8_t* dstT = a.VrT + (int64_t)bh * 128 * Np + n0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int idx = i * kPrepThreads + t;
        const int c = idx >> 3, part = idx & 7;
        *reinterpret_cast<uint4*>(dstT + (int64_t)c * Np + 16 * (part ^ (vseg_swz(c) >> 1))) =
            *reinterpret_cast<const uint4*>(codeT + c * 128 + part * 16);
      }
      }
    }
    // this warp is done with the stage (its reads and, for V, the scratch)
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stg]);
  }
  if (abort_s) {
    // let copies already issued land before the CTA exits
    for (int i = 0; i < kStreamStages; ++i) {
      int never = 0;
      mbar_wait_bounded(&full[i], 0, &never, nullptr, lim, 801);
      mbar_wait_bounded(&full[i], 1, &never, nullptr, lim, 802);
    }
  }
}



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

// The 4-bit prep's second pass over V (the first ran in the streaming
// kernel: block means in v_mean, the heads' residual maxima in head_amax).
__global__ void __launch_bounds__(kPrepThreads) smooth_quant_v4_kernel(const PrepV4Args a) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t* tile = reinterpret_cast<uint16_t*>(sm);     // [128][136] bf16
  uint8_t* codeT = sm + 128 * kTilePitch * 2;           // [128][80] u8
  __shared__ float mu_s[128];

  const int blk = blockIdx.x, bh = blockIdx.y;
  const int N = a.N, nb = a.nb;
  const int64_t Np = (int64_t)nb * 128;
  const int n0 = blk * 128;
  const int nv = min(128, N - n0);
  const int t = threadIdx.x;
  const int chunk = t & 15, rsub = t >> 4;
  const uint16_t* src = a.V + (int64_t)bh * N * 128;
  const int32_t* perm = a.perm + (int64_t)bh * N;

  // ---- gather the block's 128 permuted value rows into shared memory
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int row = it * 16 + rsub;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (row < nv) w = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)__ldg(perm + n0 + row) * 128) + chunk);
    *reinterpret_cast<uint4*>(tile + row * kTilePitch + chunk * 8) = w;
  }
  const int ch = t & 127, half = t >> 7;

  // ---- code (channel, 16-token group) units, four per thread
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

constexpr size_t kV4Smem = 128 * kTilePitch * 2 + 128 * kV4Pitch;

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
  if (cudaFuncSetAttribute(smooth_quant_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kStreamSmem) != cudaSuccess)
    return fail(VCA_ERR_CUDA, "vca_smooth_quantize_qkv: cannot set shared-memory size");
  PrepArgs a;
  a.Q = Q; a.K = K; a.V = V; a.perm = perm; a.N = N; a.nb = (N + 127) / 128;
  a.Qq = Qq; a.q_scale = q_scale; a.Kq = Kq; a.k_scale = k_scale; a.VrT = VrT;
  a.v_exp = v_exp; a.v_mean = v_mean; a.st = (DevStatus*)ws;
  a.head_amax = nullptr;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = 3ll * B * H * a.nb;
  const int grid = (int)std::min<long long>(items, 2ll * sms);   // two resident CTAs per SM
  smooth_quant_stream_kernel<<<grid, kStreamThreads, kStreamSmem, (cudaStream_t)stream>>>(a, B * H, wait_limit_ns());
  return check_launch("smooth_quant_stream_kernel");
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
  unsigned* head_amax = reinterpret_cast<unsigned*>((char*)ws + 256);
  if (cudaMemsetAsync(head_amax, 0, (size_t)B * H * 4, s) != cudaSuccess)
    return fail(VCA_ERR_CUDA, "%s: memset failed", fn);
  // Q, K (the 8-bit prep's codes) and the first pass over V (block means and
  // the heads' residual maxima) in one persistent launch of the streaming kernel
  if (cudaFuncSetAttribute(smooth_quant_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kStreamSmem) != cudaSuccess)
    return fail(VCA_ERR_CUDA, "%s: cannot set shared-memory size", fn);
  PrepArgs a;
  a.Q = Q; a.K = K; a.V = V; a.perm = perm; a.N = N; a.nb = nb;
  a.Qq = Qq; a.q_scale = q_scale; a.Kq = Kq; a.k_scale = k_scale; a.VrT = nullptr;
  a.v_exp = nullptr; a.v_mean = v_mean; a.st = (DevStatus*)ws; a.head_amax = head_amax;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)std::min<long long>(3ll * B * H * nb, 2ll * sms);
  smooth_quant_stream_kernel<<<grid, kStreamThreads, kStreamSmem, s>>>(a, B * H, wait_limit_ns());
  int rc = check_launch("smooth_quant_stream_kernel (4-bit prep)");
  if (rc) return rc;
  // the NVFP4 residual, coded with the heads' tensor scales
  PrepV4Args v;
  v.V = V; v.perm = perm; v.N = N; v.nb = nb; v.VrT4 = VrT4; v.v_sc = v_sc; v.v_gscale = v_gscale;
  v.v_mean = v_mean; v.head_amax = head_amax; v.st = (DevStatus*)ws;
  smooth_quant_v4_kernel<<<dim3(nb, B * H), kPrepThreads, kV4Smem, s>>>(v);
  return check_launch("smooth_quant_v4_kernel");
}
