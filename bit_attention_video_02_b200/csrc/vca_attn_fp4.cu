// vca_attn_fp4.cu -- attention of the 4-bit V-Smooth variant: NVFP4 values and
// probabilities in the PV product.
//
// Method ("Nunchux AI Introduces VC-Attention..." abstract: a 4-bit V-Smooth
// variant; ExpCast is 8-bit only, since NVFP4 has no single affine map from
// the log-domain score to its code; "Accelerating Video Generation with GEMM
// Quantization, Attention Quantization and Skip Softmax Attention in
// TensorRT-LLM", table of quantisation formats: NVFP4 = E2M1 elements, one
// E4M3 scale per 16 elements, one fp32 scale per tensor):
//  * QK^T as in the 8-bit path (E4M3 operands with per-block fp32 scales).
//  * Per row and key block, against the same reference maximum n (phi grid,
//    4 octaves of headroom, lag rule) as the 8-bit path, p = 2^(z - n - phi + 4)
//    in fp32, then NVFP4 per 16 keys with the fixed tensor scale 2^-3:
//      sc = e4m3(max p / 0.75), s = decode(sc) * 2^-3, code = e2m1(p * (1/s)),
//    each quotient, reciprocal and product rounded once in fp32.
//  * V residual in NVFP4 from vca_smooth_quantize_qkv_fp4 (E2M1 codes, E4M3
//    scale per 16 tokens of a channel, fp32 scale G per head).
//  * PV: tcgen05 kind::mxf4nvf4.block_scale.scale_vec::4X with A = P codes read
//    from tensor memory, the P group scales as A's UE4M3 scale factors and the
//    V group scales as B's; the accumulator holds sum p r / (2^-3 G).
//  * Mean restore: O += L (M / G) by TF32 MMAs every 8 key blocks, L the block
//    row sums of the dequantised probabilities over 2^-3 (split hi + lo), M / G
//    the bf16 block means over G (split hi + lo); the epilogue multiplies by
//    G / sum L.
// Kernel structure as the 8-bit kernel: one CTA = two 128-row query tiles of
// one head, warp 0 TMA, warp 1 MMA issuer and TMEM owner, warp 2 mean tiles,
// warps 4-7 / 8-11 the softmax warpgroups of tiles 0 / 1 (thread = row = TMEM
// lane); one score tile S in TMEM shared by the two query tiles in turn and
// released as soon as a warpgroup has loaded it.  Every wait is bounded.
#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

namespace fp4 {

constexpr int kThreads = 384;
constexpr int kStages = 3;
constexpr int kGroup = 8;   // key blocks per mean-restore MMA

// TMEM columns
constexpr uint32_t kColS = 0;     // score tile (128 columns)
// P region: tile t at +64t: the scale factors of K step k (64 keys) at +4k
// (A, the P group scales) and +8+4k (B, the V group scales), codes +16..+31.
// Scale-factor addresses are multiples of 4 columns.  In the 4 columns of one
// K step, row r's A scales (4 bytes, one per 16 keys) sit at lane r, column
// r / 32; B column n's at column n / 32 and lane 32 q + n % 32 in each of the
// four lane quarters q (measured with vca_debug_fp4_mma).
constexpr uint32_t kColP = 128;
constexpr uint32_t kColO = 256;   // O_t at +128t

// dynamic shared memory layout (offsets from a 1024-aligned base)
constexpr uint32_t kOffQ = 0;                          // 2 x 16 KB
constexpr uint32_t kOffK = 32768;                      // kStages x 16 KB
constexpr uint32_t kOffV = kOffK + kStages * 16384;    // kStages x 8 KB (128 channels x 64 bytes)
constexpr uint32_t kOffL = kOffV + kStages * 8192;     // 2 tiles x (hi 4 KB + lo 4 KB)
constexpr uint32_t kOffMu = kOffL + 16384;             // 2 buffers x (hi 4 KB + lo 4 KB)
constexpr uint32_t kSmemBytes = kOffMu + 16384;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;

constexpr float kPScale = 0.125f;   // tensor scale of the probabilities

struct Params {
  CUtensorMap tmQ, tmK, tmV;
  const float* q_scale;
  const float* k_scale;
  const uint8_t* v_sc;      // [B*H][128][Np/16] E4M3 group scales
  const float* v_gscale;    // [B*H]
  const uint16_t* v_mean;
  uint16_t* O;
  float* lse;
  int N, nb;
  float c_base;            // softmax_scale * log2(e)
  double c_base_d;         // the same in fp64
  DevStatus* st;
  unsigned long long wait_ns;
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t mu_full[2];
  uint64_t mu_empty[2];
  uint64_t mma_done;
};

__device__ __forceinline__ uint32_t tf32_off(int r, int k) {
  return (uint32_t)((r >> 3) * 256 + (k >> 2) * 128 + (r & 7) * 16 + (k & 3) * 4);
}

}  // namespace fp4

// O += A B with A (E2M1) read from tensor memory, B (E2M1) from a shared-memory
// descriptor and UE4M3 scale factors per 16 elements of K for both.
__device__ __forceinline__ void mma_nvf4_ts_w(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                              uint32_t sfa, uint32_t sfb, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], [%1], %2, %3, [%4], [%5], p;"
      "\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accum));
}

// Instruction descriptor of kind::mxf4nvf4: A and B format E2M1 (code 1 in the
// 3-bit fields at bits 7 and 10), N >> 3 at bit 17, scale format bit 23 = 0
// (UE4M3), M >> 4 at bit 24, scale-factor ids 0.
__host__ __device__ constexpr uint32_t instr_desc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Two fp32 values -> two E2M1 codes, round to nearest even, saturating at 6
// (hardware cvt): low nibble = code(lo), high nibble = code(hi).
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tmov.b16 %0, {b, 0};\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r;
}
// Two E2M1 codes (one byte) -> their values as f16x2 (exact).
__device__ __forceinline__ uint32_t dec_e2m1x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tmov.b16 {b, _}, t;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(r)
      : "r"(byte));
  return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

using namespace fp4;

__global__ void __launch_bounds__(kThreads, 1) attn_fp4_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ Bars bars;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int never_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int N = p.N, nb = p.nb, nkv = nb;
  const int ngroups = (nkv + kGroup - 1) / kGroup;
  const int64_t Np = (int64_t)nb * 128;
  const uint64_t lim = p.wait_ns;

  if (threadIdx.x == 0) {
    abort_s = 0;
    never_s = 0;
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars.kv_full[s], 1);
      mbar_init(&bars.kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars.s_full[t], 1);
      mbar_init(&bars.s_free[t], 128);
      mbar_init(&bars.p_full[t], 128);
      mbar_init(&bars.o_done[t], 1);
      mbar_init(&bars.mu_full[t], 32);
      mbar_init(&bars.mu_empty[t], 1);
    }
    mbar_init(&bars.mma_done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&p.tmQ);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
  }
  __shared__ int skip_s;
  if (threadIdx.x == 0) skip_s = (p.st && *reinterpret_cast<volatile int*>(&p.st->code) == VCA_ERR_TIMEOUT);
  __syncthreads();
  if (skip_s) return;
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars.q_full, 32768);
      const int qrow = (int)((int64_t)bh * Np) + pair * 256;
      tma_load_2d(sm + kOffQ, &p.tmQ, &bars.q_full, 0, qrow);
      tma_load_2d(sm + kOffQ + 16384, &p.tmQ, &bars.q_full, 0, qrow + 128);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % kStages, u = j / kStages;
        if (u > 0 && !mbar_wait_bounded(&bars.kv_empty[s], (u - 1) & 1, &abort_s, p.st, lim, 100)) break;
        mbar_arrive_expect_tx(&bars.kv_full[s], 16384 + 8192);
        tma_load_2d(sm + kOffK + s * 16384, &p.tmK, &bars.kv_full[s], 0, (int)((int64_t)bh * Np) + j * 128);
        tma_load_2d(sm + kOffV + s * 8192, &p.tmV, &bars.kv_full[s], j * 64, bh * 128);
        issued = j + 1;
      }
      if (abort_s) {
        for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
          mbar_wait_bounded(&bars.kv_full[j % kStages], (j / kStages) & 1, &never_s, nullptr, lim, 101);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t id_qk = instr_desc(kFmtE4M3, kFmtE4M3, 128, 128, 0, 0);
    const uint32_t id_pv = instr_desc_nvf4(128, 128);
    const uint32_t id_mu = instr_desc(kFmtTF32, kFmtTF32, 128, 128, 0, 0);
    const uint64_t dQ = smem_desc(smem_u32(sm + kOffQ), 16, 1024, kLayoutSW128);
    const uint64_t dK = smem_desc(smem_u32(sm + kOffK), 16, 1024, kLayoutSW128);
    // V tile: 128 channel rows of 64 bytes (128 E2M1 tokens), 64-byte swizzle,
    // 8-row groups 512 bytes apart; +2 (32 bytes, 64 tokens) per K step, +512
    // (8 KB) per stage
    const uint64_t dV = smem_desc(smem_u32(sm + kOffV), 16, 512, kLayoutSW64);
    const uint64_t dL = smem_desc(smem_u32(sm + kOffL), 128, 256, kLayoutNone);
    const uint64_t dMu = smem_desc(smem_u32(sm + kOffMu), 128, 256, kLayoutNone);
    const uint32_t tS = tmem + kColS;
    auto issue_qk = [&](int t, int jj) {
      const int s1 = jj % kStages;
      VCA_MMA4_SS_W("f8f6f4", tS, dQ + (uint64_t)(t * 1024), dK + (uint64_t)(s1 * 1024), id_qk, 0u, &bars.s_full[t]);
    };
    auto issue_pv = [&](int t, int j) -> bool {
      if (!mbar_wait_warp(&bars.p_full[t], j & 1, &abort_s, p.st, lim, 210 + t)) return false;
      tc_fence_after();
      const int s = j % kStages;
      const uint32_t tP = tmem + kColP + t * 64;
#pragma unroll
      for (int k = 0; k < 2; ++k)   // 64 keys per K step: 8 code columns, one scale column each
        mma_nvf4_ts_w(tmem + kColO + t * 128, tP + 16 + 8 * k, dV + (uint64_t)(s * 512 + 2 * k), id_pv, tP + 4 * k,
                      tP + 8 + 4 * k, (j > 0 || k > 0) ? 1u : 0u);
      const bool group_end = (j % kGroup == kGroup - 1) || (j == nkv - 1);
      if (group_end) {
        const int g = j / kGroup, gb = g & 1;
        if (!mbar_wait_warp(&bars.mu_full[gb], (g >> 1) & 1, &abort_s, p.st, lim, 220)) return false;
        tc_fence_after();
        const uint64_t mhi = dMu + (uint64_t)(gb * 512), mlo = mhi + 256;
        const uint64_t lhi = dL + (uint64_t)(t * 512), llo = lhi + 256;
        const uint32_t d = tmem + kColO + t * 128;
        mma_tf32_ss_w(d, lhi, mhi, id_mu, 1u);
        mma_tf32_ss_w(d, lhi, mlo, id_mu, 1u);
        mma_tf32_ss_w(d, llo, mhi, id_mu, 1u);
        if (t == 1) tc_commit_w(&bars.mu_empty[gb]);
      }
      tc_commit_w(&bars.o_done[t]);
      return true;
    };
    bool ok = mbar_wait_warp(&bars.q_full, 0, &abort_s, p.st, lim, 200);
    ok = ok && mbar_wait_warp(&bars.kv_full[0], 0, &abort_s, p.st, lim, 201);
    if (ok) {
      tc_fence_after();
      issue_qk(0, 0);
    }
    ok = ok && mbar_wait_warp(&bars.s_free[0], 0, &abort_s, p.st, lim, 202);
    if (ok) {
      tc_fence_after();
      issue_qk(1, 0);
    }
    if (ok && nkv > 1) {
      ok = mbar_wait_warp(&bars.s_free[1], 0, &abort_s, p.st, lim, 203) &&
           mbar_wait_warp(&bars.kv_full[1 % kStages], (1 / kStages) & 1, &abort_s, p.st, lim, 204);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 1);
      }
    }
    for (int j = 0; ok && j < nkv; ++j) {
      ok = issue_pv(0, j);
      if (!ok) break;
      if (j + 1 < nkv) {
        ok = mbar_wait_warp(&bars.s_free[0], (j + 1) & 1, &abort_s, p.st, lim, 230);
        if (!ok) break;
        tc_fence_after();
        issue_qk(1, j + 1);
      }
      ok = issue_pv(1, j);
      if (!ok) break;
      tc_commit_w(&bars.kv_empty[j % kStages]);
      if (j + 2 < nkv) {
        const int s2 = (j + 2) % kStages;
        ok = mbar_wait_warp(&bars.s_free[1], (j + 1) & 1, &abort_s, p.st, lim, 231) &&
             mbar_wait_warp(&bars.kv_full[s2], ((j + 2) / kStages) & 1, &abort_s, p.st, lim, 232);
        if (!ok) break;
        tc_fence_after();
        issue_qk(0, j + 2);
      }
    }
    tc_commit_w(&bars.mma_done);
  } else if (warp == 2) {
    // ------------------------------------------------------------ mean tiles M / G (hi + lo), fp32 [d][8]
    const uint16_t* vm = p.v_mean + (int64_t)bh * nb * 128;
    const float G = __ldg(p.v_gscale + bh);
    for (int g = 0; g < ngroups; ++g) {
      const int gb = g & 1, u = g >> 1;
      if (u > 0 && !mbar_wait_bounded(&bars.mu_empty[gb], (u - 1) & 1, &abort_s, p.st, lim, 300)) break;
      uint8_t* dst = sm + kOffMu + gb * 8192;
      for (int q = 0; q < 4; ++q) {
        const int dch = q * 32 + lane;
        for (int kk = 0; kk < kGroup; ++kk) {
          const int blk = g * kGroup + kk;
          const float mu = blk < nb ? __uint_as_float((uint32_t)__ldg(vm + (int64_t)blk * 128 + dch) << 16) : 0.0f;
          const float x = __fdiv_rn(mu, G);
          const float hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
          *reinterpret_cast<float*>(dst + tf32_off(dch, kk)) = hi;
          *reinterpret_cast<float*>(dst + 4096 + tf32_off(dch, kk)) = x - hi;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars.mu_full[gb]);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp >> 2) - 1;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + kColS + lane_off;
    const uint32_t tP = tmem + kColP + t * 64 + lane_off;
    const uint32_t tO = tmem + kColO + t * 128 + lane_off;
    const int qtile = pair * 2 + t;
    const bool qvalid = qtile < nb;
    const float sq = !qvalid ? 1.0f : __ldg(p.q_scale + (int64_t)bh * nb + qtile);
    const float cq = sq * p.c_base;
    uint8_t* sLt = sm + kOffL + t * 8192;
    const float* ksc = p.k_scale + (int64_t)bh * nb;
    // V group scales: lane i of every warp writes those of channels i, 32+i,
    // 64+i, 96+i (B's scale columns are replicated across the lane quarters)
    const int q = warp & 3;
    const uint2* vsc = reinterpret_cast<const uint2*>(p.v_sc + ((int64_t)bh * 128 + lane) * (Np / 16));
    const int64_t vcs = 32 * (Np / 16) / 8;   // uint2 stride of 32 channels
    int nref = 0;
    float ltot = 0.0f;
    bool ok = true;
    float ksc_next = __ldg(ksc);
    uint2 vsc_next[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) vsc_next[c] = __ldg(vsc + c * vcs);
    for (int j = 0; j < nkv; ++j) {
      const float ksc_j = ksc_next;
      uint2 vsc_j[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) vsc_j[c] = vsc_next[c];
      if (j + 1 < nkv) {
        ksc_next = __ldg(ksc + j + 1);
#pragma unroll
        for (int c = 0; c < 4; ++c) vsc_next[c] = __ldg(vsc + c * vcs + j + 1);
      }
      ok = mbar_wait_warp(&bars.s_full[t], j & 1, &abort_s, p.st, lim, 400 + t);
      if (!ok) break;
      tc_fence_after();
      float sv[128];
      {
        uint32_t* su = reinterpret_cast<uint32_t*>(sv);
        VCA_TMEM_LD32(tS + 0, (su + 0));
        VCA_TMEM_LD32(tS + 32, (su + 32));
        VCA_TMEM_LD32(tS + 64, (su + 64));
        VCA_TMEM_LD32(tS + 96, (su + 96));
        tmem_ld_wait();
      }
      tc_fence_before();
      mbar_arrive(&bars.s_free[t]);
      const int valid = min(128, N - j * 128);
      if (valid < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) sv[c] = -INFINITY;
      }
      float mq[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float m = sv[32 * q];
#pragma unroll
        for (int i = 1; i < 31; i += 2) m = fmax3(m, sv[32 * q + i], sv[32 * q + i + 1]);
        mq[q] = fmaxf(m, sv[32 * q + 31]);
      }
      const float mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
      const float cz = cq * ksc_j;
      // the exponent's multiplier as an fp32 pair (hi + lo = the fp64 product):
      // a code step of E2M1 is up to half the value, so the fp32 rounding of
      // q_scale * k_scale * scale * log2(e) would flip codes at long sequences
      const double czd = (double)sq * p.c_base_d * (double)ksc_j;
      const float cz_hi = (float)czd, cz_lo = (float)(czd - (double)cz_hi);
      const int ntile = (int)ceilf(__fmaf_rn(mx, cz, -0.08125f));
      float rescale = 1.0f;
      if (j == 0) {
        nref = ntile;
      } else if (ntile > nref + 4) {
        const int delta = ntile - nref;
        nref = ntile;
        rescale = delta > 126 ? 0.0f : __uint_as_float((uint32_t)(127 - delta) << 23);
      }
      // p = 2^(z - n - phi + 4), NVFP4 per 16 keys; the row sum adds the
      // dequantised values over 2^-3: sum_g decode(sc_g) * sum_i e2m1(code_i)
      const float bias = 3.91875f - (float)nref;   // 4 - phi - n
      uint32_t pw[16];   // 128 E2M1 codes, 8 per word, in key order
      uint32_t sfa[2];   // the 8 group scale codes, 4 per word
      float l = 0.0f;
      const float2 czh2 = make_float2(cz_hi, cz_hi), czl2 = make_float2(cz_lo, cz_lo);
      const float2 bias2 = make_float2(bias, bias);
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float pv[16];
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          // z - n - phi + 4 with z = s (cz_hi + cz_lo): the product's rounding
          // error recovered by an fma, the small terms added last (two scores
          // per f32x2 instruction, each element rounded as the scalar form)
          const float2 s2 = make_float2(sv[16 * g + i], sv[16 * g + i + 1]);
          const float2 zh = __fmul2_rn(s2, czh2);
          const float2 zl = __ffma2_rn(s2, czl2, __ffma2_rn(s2, czh2, make_float2(-zh.x, -zh.y)));
          const float2 a = __fadd2_rn(__fadd2_rn(zh, bias2), zl);
          pv[i] = ex2_approx(a.x);
          pv[i + 1] = ex2_approx(a.y);
          if (valid < 128) {   // keys past the end (the error term is NaN there)
            if (16 * g + i >= valid) pv[i] = 0.0f;
            if (16 * g + i + 1 >= valid) pv[i + 1] = 0.0f;
          }
          am = fmax3(am, pv[i], pv[i + 1]);
        }
        const uint32_t sc = cvt_e4m3x2(__fdiv_rn(am, 0.75f), 0.0f) & 0xFFu;
        const float s = __uint_as_float(sc << 20) * 0x1p120f;   // decode(sc), exact
        const float sg = s * kPScale;
        uint32_t w0 = 0u, w1 = 0u;
        float gsum = 0.0f;
        if (sg > 0.0f) {
          const float inv = __frcp_rn(sg);
          uint32_t b[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 y = __fmul2_rn(make_float2(pv[2 * i], pv[2 * i + 1]), make_float2(inv, inv));
            b[i] = cvt_e2m1x2(y.x, y.y);
          }
          w0 = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
          w1 = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
          __half2 acc = __halves2half2(__float2half_rn(0.0f), __float2half_rn(0.0f));
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t h = dec_e2m1x2(b[i]);
            acc = __hadd2(acc, *reinterpret_cast<const __half2*>(&h));   // exact: sums <= 96 in steps of 0.5
          }
          gsum = (__low2float(acc) + __high2float(acc)) * s;   // exact
        }
        pw[2 * g] = w0;
        pw[2 * g + 1] = w1;
        if ((g & 3) == 0) sfa[g >> 2] = 0u;
        sfa[g >> 2] |= sc << (8 * (g & 3));
        l += gsum;
      }
      // PV(j-1) and the mean restore issued with it must have completed
      // before the P region, sL_t or O_t are written
      if (j > 0) {
        ok = mbar_wait_warp(&bars.o_done[t], (j - 1) & 1, &abort_s, p.st, lim, 410 + t);
        if (!ok) break;
        tc_fence_after();
      }
      const int kk = j % kGroup;
      {
        const float hi = __uint_as_float(__float_as_uint(l) & 0xFFFFE000u);
        *reinterpret_cast<float*>(sLt + tf32_off(r, kk)) = hi;
        *reinterpret_cast<float*>(sLt + 4096 + tf32_off(r, kk)) = l - hi;
        if (j == nkv - 1) {
          for (int k2 = kk + 1; k2 < kGroup; ++k2) {
            *reinterpret_cast<float*>(sLt + tf32_off(r, k2)) = 0.0f;
            *reinterpret_cast<float*>(sLt + 4096 + tf32_off(r, k2)) = 0.0f;
          }
        }
      }
      VCA_TMEM_ST16(tP + 16, pw);
      {
        // scale factors (bytes = 16-key groups in key order): this row's P
        // group scales in the column of its lane quarter, and the V group
        // scales of channels 32c + lane in column c
        uint32_t sf[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          sf[c] = c == q ? sfa[0] : 0u;
          sf[4 + c] = c == q ? sfa[1] : 0u;
          sf[8 + c] = vsc_j[c].x;
          sf[12 + c] = vsc_j[c].y;
        }
        VCA_TMEM_ST16(tP, sf);   // columns +0..+15
      }
      if (__any_sync(0xffffffffu, rescale != 1.0f)) {
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t o[32];
          VCA_TMEM_LD32(tO + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * rescale);
          VCA_TMEM_ST32(tO + c0, o);
        }
        for (int k2 = 0; k2 < kk; ++k2) {
          float* hp = reinterpret_cast<float*>(sLt + tf32_off(r, k2));
          float* lp = reinterpret_cast<float*>(sLt + 4096 + tf32_off(r, k2));
          *hp *= rescale;
          *lp *= rescale;
        }
      }
      ltot = ltot * rescale + l;
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars.p_full[t]);
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = mbar_wait_warp(&bars.o_done[t], (nkv - 1) & 1, &abort_s, p.st, lim, 420 + t);
    if (ok) {
      tc_fence_after();
      const int qrow = qtile * 128 + r;
      const bool store = qvalid && qrow < N;
      const float f = __fdiv_rn(__ldg(p.v_gscale + bh), ltot);   // G / sum L
      uint16_t* orow = p.O + ((int64_t)bh * N + qrow) * 128;
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t o[32];
        VCA_TMEM_LD32(tO + c0, o);
        tmem_ld_wait();
        if (store) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(o[2 * c]) * f, __uint_as_float(o[2 * c + 1]) * f);
            pk[c] = *reinterpret_cast<uint32_t*>(&hv);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      // ln of the decoded probabilities' sum: (n + phi - 4) + log2(2^-3 sum L)
      if (store && p.lse)
        p.lse[(int64_t)bh * N + qrow] = 0.69314718055994531f * ((float)nref + 0.08125f - 7.0f + __log2f(ltot));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    mbar_wait_bounded(&bars.mma_done, 0, &never_s, nullptr, lim, 500);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One CTA, one 128x128x128 product through the same block-scaled FP4 MMA as
// the attention kernel: A codes at tensor-memory columns 16..31, the 16 scale
// columns 0..15 as given (SFA of K step k at column 4k, SFB at 8 + 4k), B by
// TMA in the 64-byte swizzled layout.  Known operands in, D out: a check of
// the operand and scale-factor layouts.
__global__ void __launch_bounds__(128, 1) fp4_mma_check_kernel(const __grid_constant__ CUtensorMap tmB,
                                                               const uint32_t* a_words, const uint32_t* sf_words,
                                                               float* D, DevStatus* st, unsigned long long lim) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full, done;
  __shared__ uint32_t tbase;
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5, r = threadIdx.x;
  if (r == 0) {
    abort_s = 0;
    mbar_init(&full, 1);
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tbase, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  if (r == 0) {
    mbar_arrive_expect_tx(&full, 8192);
    tma_load_2d(sm, &tmB, &full, 0, 0);
  }
  // row r: 16 code words, 2 SFA words, 2 SFB words (SFB row r = B column r)
  // (the same column layout as the attention kernel's P region)
  uint32_t a[16], sf[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = a_words[r * 16 + i];
#pragma unroll
  for (int i = 0; i < 16; ++i) sf[i] = sf_words[r * 16 + i];
  VCA_TMEM_ST16(tmem + 16 + lane_off, a);
  VCA_TMEM_ST16(tmem + lane_off, sf);
  tmem_st_wait();
  tc_fence_before();
  __syncthreads();
  bool ok = true;
  if (warp == 0) {
    ok = mbar_wait_warp(&full, 0, &abort_s, st, lim, 700);
    if (ok) {
      tc_fence_after();
      const uint64_t dB = smem_desc(smem_u32(sm), 16, 512, kLayoutSW64);
#pragma unroll
      for (int k = 0; k < 2; ++k)
        mma_nvf4_ts_w(tmem + 128, tmem + 16 + 8 * k, dB + (uint64_t)(2 * k), instr_desc_nvf4(128, 128), tmem + 4 * k,
                      tmem + 8 + 4 * k, k > 0 ? 1u : 0u);
    }
    tc_commit_w(&done);
  }
  ok = mbar_wait_bounded(&done, 0, &abort_s, st, lim, 701) && ok;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  if (ok) {
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t o[32];
      VCA_TMEM_LD32(tmem + 128 + c0 + lane_off, o);
      tmem_ld_wait();
      for (int c = 0; c < 32; ++c) D[r * 128 + c0 + c] = __uint_as_float(o[c]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace vca

using namespace vca;

extern "C" int vca_attention_fwd_fp4(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq, const float* k_scale,
                                     const uint8_t* VrT4, const uint8_t* v_sc, const float* v_gscale,
                                     const vca_bf16* v_mean, int B, int H, int N, int d, float softmax_scale,
                                     vca_bf16* O, float* lse, void* ws, size_t ws_bytes, vca_stream_t stream) {
  const char* fn = "vca_attention_fwd_fp4";
  if (d != VCA_HEAD_DIM) return fail(VCA_ERR_UNSUPPORTED, "%s: d must be 128", fn);
  if (B < 1 || H < 1 || N < 1 || (int64_t)B * H > 65535)
    return fail(VCA_ERR_INVALID, "%s: bad shape B=%d H=%d N=%d", fn, B, H, N);
  const int nb = (N + 127) / 128;
  const int64_t Np = (int64_t)nb * 128;
  if ((int64_t)B * H * Np > INT32_MAX || Np > INT32_MAX / 2)
    return fail(VCA_ERR_UNSUPPORTED, "%s: B*H*Np exceeds the 2^31 row limit", fn);
  const void* ptrs[] = {Qq, q_scale, Kq, k_scale, VrT4, v_sc, v_gscale, v_mean, O};
  for (const void* q : ptrs)
    if (!q) return fail(VCA_ERR_INVALID, "%s: null pointer", fn);
  const void* al[] = {Qq, Kq, VrT4, O};
  for (const void* q : al)
    if (!aligned16(q)) return fail(VCA_ERR_INVALID, "%s: tensors must be 16-byte aligned", fn);
  if ((reinterpret_cast<uintptr_t>(v_sc) & 7u) != 0)
    return fail(VCA_ERR_INVALID, "%s: v_sc must be 8-byte aligned", fn);
  if (!(softmax_scale > 0.0f)) return fail(VCA_ERR_INVALID, "%s: softmax_scale must be > 0", fn);
  if (!ws || ws_bytes < vca_attention_workspace_size(B, H, N))
    return fail(VCA_ERR_WORKSPACE, "%s: workspace too small", fn);

  fp4::Params prm;
  const uint64_t BH = (uint64_t)B * H;
  {
    uint64_t dims[2] = {128, BH * (uint64_t)Np}, str[1] = {128};
    uint32_t box[2] = {128, 128};
    int rc = encode_tiled(&prm.tmQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, Qq, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!rc) rc = encode_tiled(&prm.tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, Kq, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    // VrT4 rows: 128 channels per head, Np/2 bytes each; a box is one block's 64 bytes x 128 channels
    uint64_t vd[2] = {(uint64_t)Np / 2, BH * 128}, vs[1] = {(uint64_t)Np / 2};
    uint32_t vbox[2] = {64, 128};
    if (!rc) rc = encode_tiled(&prm.tmV, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, VrT4, vd, vs, vbox, CU_TENSOR_MAP_SWIZZLE_64B);
    if (rc) return rc;
  }
  prm.q_scale = q_scale;
  prm.k_scale = k_scale;
  prm.v_sc = v_sc;
  prm.v_gscale = v_gscale;
  prm.v_mean = v_mean;
  prm.O = O;
  prm.lse = lse;
  prm.N = N;
  prm.nb = nb;
  prm.c_base = (float)((double)softmax_scale * 1.4426950408889634);
  prm.c_base_d = (double)softmax_scale * 1.4426950408889634;
  prm.st = (DevStatus*)ws;
  prm.wait_ns = wait_limit_ns();
  if (cudaFuncSetAttribute(attn_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fp4::kSmemAlloc) !=
      cudaSuccess)
    return fail(VCA_ERR_CUDA, "%s: cannot set shared-memory size", fn);
  dim3 grid((nb + 1) / 2, (unsigned)BH);
  attn_fp4_kernel<<<grid, fp4::kThreads, fp4::kSmemAlloc, (cudaStream_t)stream>>>(prm);
  return check_launch("attn_fp4_kernel");
}

extern "C" int vca_debug_fp4_mma(const uint8_t* a_codes, const uint8_t* sf_cols, const uint8_t* b_codes, float* D,
                                 void* ws, vca_stream_t stream) {
  const char* fn = "vca_debug_fp4_mma";
  const void* ptrs[] = {a_codes, sf_cols, b_codes, D, ws};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return fail(VCA_ERR_INVALID, "%s: null or misaligned pointer", fn);
  CUtensorMap tmB;
  uint64_t dims[2] = {64, 128}, str[1] = {64};
  uint32_t box[2] = {64, 128};
  int rc = encode_tiled(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b_codes, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc) return rc;
  if (cudaFuncSetAttribute(fp4_mma_check_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 8192 + 1024) !=
      cudaSuccess)
    return fail(VCA_ERR_CUDA, "%s: cannot set shared-memory size", fn);
  fp4_mma_check_kernel<<<1, 128, 8192 + 1024, (cudaStream_t)stream>>>(
      tmB, reinterpret_cast<const uint32_t*>(a_codes), reinterpret_cast<const uint32_t*>(sf_cols), D,
      (DevStatus*)ws, wait_limit_ns());
  return check_launch("fp4_mma_check_kernel");
}
