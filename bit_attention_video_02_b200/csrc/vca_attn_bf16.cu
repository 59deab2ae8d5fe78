// vca_attn_bf16.cu -- BF16 flash attention on tcgen05: the in-repo comparator
// for the FP8 path (exact softmax with an fp32 exp2 per score, bf16 P, fp32
// accumulation in tensor memory).
//
// Same CTA organisation as the FP8 kernel: two 128-row query tiles per CTA,
// warp 0 loads (TMA, 128B swizzle, two 64-channel boxes per tile), warp 1
// issues MMAs, warps 4-7 / 8-11 run the softmax of query tile 0 / 1.
//  * S_t = Q_t K_j^T: kind::f16, both operands K-major in shared memory.
//  * P_t (bf16) is stored into the consumed S_t columns (64 columns) and fed
//    back from tensor memory; V is the MN-major B operand, so O_t += P_t V_j
//    needs no transpose.
//  * Online softmax with lazy rescale: O and the row sum are rescaled only when
//    the running maximum grows by more than 8 (log2 units).
#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

constexpr int kBfThreads = 384;
constexpr int kBfStages = 2;
constexpr uint32_t kBfOffQ = 0;                              // 2 tiles x 32 KB
constexpr uint32_t kBfOffK = 65536;                          // stages x 32 KB
constexpr uint32_t kBfOffV = kBfOffK + kBfStages * 32768;    // stages x 32 KB
constexpr uint32_t kBfSmem = kBfOffV + kBfStages * 32768 + 1024;

struct BfParams {
  CUtensorMap tmQ, tmK, tmV;
  uint16_t* O;
  float* lse;
  int N, nt;
  float c_base;   // softmax_scale * log2(e)
  DevStatus* st;
  unsigned long long wait_ns;
};

struct __align__(8) BfBars {
  uint64_t q_full;
  uint64_t kv_full[kBfStages];
  uint64_t kv_empty[kBfStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t mma_done;
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kBfThreads, 1) attn_bf16_kernel(const __grid_constant__ BfParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ BfBars bars;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s, never_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int N = p.N, nkv = p.nt;
  const uint64_t lim = p.wait_ns;

  if (threadIdx.x == 0) {
    abort_s = 0;
    never_s = 0;
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kBfStages; ++s) {
      mbar_init(&bars.kv_full[s], 1);
      mbar_init(&bars.kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars.s_full[t], 1);
      mbar_init(&bars.p_full[t], 128);
      mbar_init(&bars.o_done[t], 1);
    }
    mbar_init(&bars.mma_done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&p.tmQ);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
  }
  // a CTA of this launch (or of an earlier one sharing the workspace) already
  // timed out: do no work, so a broken pipeline costs one wait, not one per CTA
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
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars.q_full, 65536);
      for (int t = 0; t < 2; ++t)
        for (int h = 0; h < 2; ++h)
          tma_load_3d(sm + kBfOffQ + t * 32768 + h * 16384, &p.tmQ, &bars.q_full, h * 64,
                      pair * 256 + t * 128, bh);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % kBfStages, u = j / kBfStages;
        if (u > 0 && !mbar_wait_bounded(&bars.kv_empty[s], (u - 1) & 1, &abort_s, p.st, lim, 100)) break;
        mbar_arrive_expect_tx(&bars.kv_full[s], 65536);
        for (int h = 0; h < 2; ++h) {
          tma_load_3d(sm + kBfOffK + s * 32768 + h * 16384, &p.tmK, &bars.kv_full[s], h * 64, j * 128, bh);
          tma_load_3d(sm + kBfOffV + s * 32768 + h * 16384, &p.tmV, &bars.kv_full[s], h * 64, j * 128, bh);
        }
        issued = j + 1;
      }
      if (abort_s)
        for (int j = (issued > kBfStages ? issued - kBfStages : 0); j < issued; ++j)
          mbar_wait_bounded(&bars.kv_full[j % kBfStages], (j / kBfStages) & 1, &never_s, nullptr, lim, 101);
    }
  } else if (warp == 1) {
    // the whole warp runs the issue loop (warp-uniform descriptors advanced by
    // constants); one elected lane issues each tcgen05 instruction
    const uint32_t id_qk = instr_desc(kFmtBF16, kFmtBF16, 128, 128, 0, 0);
    const uint32_t id_pv = instr_desc(kFmtBF16, kFmtBF16, 128, 128, 0, 1);
    // descriptor start addresses count 16-byte units
    const uint64_t dQ = smem_desc(smem_u32(sm + kBfOffQ), 16, 1024, kLayoutSW128);
    const uint64_t dK = smem_desc(smem_u32(sm + kBfOffK), 16, 1024, kLayoutSW128);
    const uint64_t dV = smem_desc(smem_u32(sm + kBfOffV), 16384, 1024, kLayoutSW128);
    bool ok = mbar_wait_warp(&bars.q_full, 0, &abort_s, p.st, lim, 200);
    ok = ok && mbar_wait_warp(&bars.kv_full[0], 0, &abort_s, p.st, lim, 201);
    auto issue_qk = [&](int t, int s) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint64_t off = (uint64_t)((k >> 2) * 1024 + (k & 3) * 2);   // (k/4)*16 KB + (k%4)*32 B
        mma_bf16_ss_w(tmem + t * 128, dQ + (uint64_t)(t * 2048) + off, dK + (uint64_t)(s * 2048) + off, id_qk,
                      k > 0);
      }
      tc_commit_w(&bars.s_full[t]);
    };
    if (ok) {
      tc_fence_after();
      issue_qk(0, 0);
      issue_qk(1, 0);
    }
    for (int j = 0; ok && j < nkv; ++j) {
      const int s = j % kBfStages;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        ok = mbar_wait_warp(&bars.p_full[t], j & 1, &abort_s, p.st, lim, 210 + t);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_bf16_ts_w(tmem + 256 + t * 128, tmem + t * 128 + 8 * k, dV + (uint64_t)(s * 2048 + k * 128), id_pv,
                        (j > 0 || k > 0) ? 1u : 0u);
        tc_commit_w(&bars.o_done[t]);
        if (t == 1) tc_commit_w(&bars.kv_empty[s]);
        if (j + 1 < nkv) {
          const int s1 = (j + 1) % kBfStages;
          if (t == 0) {
            ok = mbar_wait_warp(&bars.kv_full[s1], ((j + 1) / kBfStages) & 1, &abort_s, p.st, lim, 230);
            if (!ok) break;
            tc_fence_after();
          }
          issue_qk(t, s1);
        }
      }
    }
    tc_commit_w(&bars.mma_done);
  } else if (warp >= 4) {
    const int t = (warp >> 2) - 1;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + t * 128 + lane_off;
    const uint32_t tO = tmem + 256 + t * 128 + lane_off;
    const int qrow = pair * 256 + t * 128 + r;
    const float cz = p.c_base;
    float mref = -INFINITY;   // running reference maximum (log2 units)
    float ltot = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
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
      const int valid = min(128, N - j * 128);
      if (valid < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) sv[c] = -INFINITY;
      }
      float mx = sv[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, sv[c]);
      const float mtile = mx * cz;
      float rescale = 1.0f;
      if (mtile > mref + 8.0f) {
        const float mnew = mtile;
        rescale = ex2_approx(mref - mnew);   // 0 on the first tile
        mref = mnew;
      }
      if (j > 0) {
        ok = mbar_wait_warp(&bars.o_done[t], (j - 1) & 1, &abort_s, p.st, lim, 410 + t);
        if (!ok) break;
        tc_fence_after();
      }
      const float nm = -mref;
      float lsum = 0.0f;
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float p0 = ex2_approx(__fmaf_rn(sv[c0 + 2 * c], cz, nm));
          const float p1 = ex2_approx(__fmaf_rn(sv[c0 + 2 * c + 1], cz, nm));
          lsum += p0 + p1;
          __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
          pk[c] = *reinterpret_cast<uint32_t*>(&h);
        }
        VCA_TMEM_ST16(tS + c0 / 2, pk);
      }
      // tcgen05.ld/st are warp-collective: the whole warp rescales if any row must
      if (j > 0 && __any_sync(0xffffffffu, rescale != 1.0f)) {
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t o[32];
          VCA_TMEM_LD32(tO + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * rescale);
          VCA_TMEM_ST32(tO + c0, o);
        }
      }
      ltot = (j > 0 ? ltot * rescale : 0.0f) + lsum;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars.p_full[t]);
    }
    if (ok) ok = mbar_wait_warp(&bars.o_done[t], (nkv - 1) & 1, &abort_s, p.st, lim, 420 + t);
    if (ok) {
      tc_fence_after();
      const bool store = qrow < N;
      const float inv = 1.0f / ltot;
      uint16_t* orow = p.O + ((int64_t)bh * N + qrow) * 128;
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t o[32];
        VCA_TMEM_LD32(tO + c0, o);
        tmem_ld_wait();
        if (store) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(o[2 * c]) * inv,
                                                     __uint_as_float(o[2 * c + 1]) * inv);
            pk[c] = *reinterpret_cast<uint32_t*>(&h);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      if (store && p.lse) p.lse[(int64_t)bh * N + qrow] = 0.69314718055994531f * (mref + __log2f(ltot));
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

}  // namespace vca

using namespace vca;

extern "C" size_t vca_bf16_attention_workspace_size(int B, int H, int N) { return 256; }

extern "C" int vca_bf16_attention_fwd(const vca_bf16* Q, const vca_bf16* K, const vca_bf16* V, int B, int H,
                                      int N, int d, float softmax_scale, vca_bf16* O, float* lse, void* ws,
                                      size_t ws_bytes, vca_stream_t stream) {
  if (d != VCA_HEAD_DIM) return fail(VCA_ERR_UNSUPPORTED, "vca_bf16_attention_fwd: d must be 128");
  if (B < 1 || H < 1 || N < 1 || (int64_t)B * H > 65535 || N > (1 << 30))
    return fail(VCA_ERR_INVALID, "vca_bf16_attention_fwd: bad shape B=%d H=%d N=%d", B, H, N);
  if (!Q || !K || !V || !O) return fail(VCA_ERR_INVALID, "vca_bf16_attention_fwd: null pointer");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(VCA_ERR_INVALID, "vca_bf16_attention_fwd: tensors must be 16-byte aligned");
  if (!(softmax_scale > 0.0f)) return fail(VCA_ERR_INVALID, "vca_bf16_attention_fwd: softmax_scale must be > 0");
  if (!ws || ws_bytes < vca_bf16_attention_workspace_size(B, H, N))
    return fail(VCA_ERR_WORKSPACE, "vca_bf16_attention_fwd: workspace too small");
  BfParams prm;
  const uint64_t BH = (uint64_t)B * H;
  uint64_t dims[3] = {128, (uint64_t)N, BH}, str[2] = {256, (uint64_t)N * 256};
  uint32_t box[3] = {64, 128, 1};
  int rc = encode_tiled(&prm.tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Q, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc) rc = encode_tiled(&prm.tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, K, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc) rc = encode_tiled(&prm.tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  prm.O = O;
  prm.lse = lse;
  prm.N = N;
  prm.nt = (N + 127) / 128;
  prm.c_base = (float)((double)softmax_scale * 1.4426950408889634);
  prm.st = (DevStatus*)ws;
  prm.wait_ns = wait_limit_ns();
  if (cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBfSmem) !=
      cudaSuccess)
    return fail(VCA_ERR_CUDA, "vca_bf16_attention_fwd: cannot set shared-memory size");
  dim3 grid((prm.nt + 1) / 2, (unsigned)BH);
  attn_bf16_kernel<<<grid, kBfThreads, kBfSmem, (cudaStream_t)stream>>>(prm);
  return check_launch("attn_bf16_kernel");
}
