// vca_attn_fp8.cu -- ExpCast-FP8 flash attention with V-Smooth mean restore.
//
// Method ("VC-Attention: Training-Free Low-Bit Attention Speeds Video
// Diffusion Up to 3.6x", V-Smooth and ExpCast-FP8 bullets; "Nunchux AI
// Introduces VC-Attention..." abstract; "VC-Attention", aikraft.ru, "Решение"):
// QK^T and PV run on 8-bit tensor cores; the softmax writes each E4M3
// probability byte from the log-domain score with one FMA (byte ~ 8 log2 p + 56
// + beta, beta = -0.35) instead of an fp32 exp2 and a cast; the value block
// mean that prep subtracted is restored from the per-block row sums.
//
// Design (sm_100a):
//  * one CTA = two 128-row query tiles of one head (they share every K/V tile);
//    12 warps: warp 0 TMA producer, warp 1 MMA issuer (the whole warp runs the
//    issue loop, one elected lane issues) and TMEM owner, warp 2 stages block
//    means, warps 4-7 / 8-11 are the softmax warpgroups of query tile 0 / 1
//    (thread = query row = TMEM lane).
//  * TMEM (512 columns): S (one fp32 score tile, shared by the two query
//    tiles in turn), O0, O1 (fp32 accumulators of 144 columns: the 128 output
//    channels and the block row sum), per tile 32 columns of packed E4M3 codes,
//    and the UE8M0 scale vectors (A's shared, B's double-buffered by key block).
//  * S = Q_t K_j^T: tcgen05 kind::f8f6f4, operands from 128B-swizzled smem.
//    A softmax warpgroup releases S as soon as it has loaded its scores into
//    registers, and the MMA warp refills it for the other tile, so the tensor
//    core computes one tile's scores while both warpgroups compute codes: the
//    two tiles run staggered by one QK^T, and the time per key block is the
//    softmax's, not softmax + MMAs.  The order of issue is
//      QK0(0) QK1(0) QK0(1) | PV0(j) QK1(j+1) PV1(j) QK0(j+2) | ...
//  * O_t += P_t R_j * 2^e_j: kind::mxf8f6f4.block_scale with A = P_t read
//    from tensor memory (no shared-memory round trip for the probabilities);
//    the per-block V exponent is the UE8M0 scale of B (A's scale is 1).  B has
//    144 rows: the V tile and a constant row of E4M3 ones (scale 2^0), so the
//    same MMAs leave the block row sum of the decoded codes in column 128 of
//    O_t, which the warpgroup reads and zeroes while coding the next block.  A
//    warpgroup writes P_t(j) and the scale vectors only after PV_t(j-1) has
//    completed (o_done), which it needs anyway before rescaling O_t.
//  * Mean restore: every 8 key blocks, O_t += L_t M^T with a TF32 MMA, where
//    L_t[i][b] are the block row sums (split hi + lo so they keep ~22 bits) and
//    M[d][b] the bf16 block means (exact in TF32).
//  * Online maximum on the grid phi + integers (phi = 0.65/8): a lagging
//    maximum changes codes by multiples of 8, i.e. probabilities by exact
//    powers of two, and O is rescaled by exact powers of two only when the
//    block maximum overtakes the reference by more than 4 octaves.  Codes are
//    written 4 octaves above the reference (row max at codes 80..88), keeping
//    the largest code at 120 < 126.
//  * Every mbarrier wait is bounded (globaltimer); on expiry the CTA records
//    VCA_ERR_TIMEOUT in the status word, all roles drain and exit, and TMEM is
//    freed after the issued MMAs complete.
#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

constexpr int kAttnThreads = 384;
constexpr int kStages = 3;
constexpr int kGroup = 8;   // key blocks per mean-restore MMA

// TMEM columns
constexpr uint32_t kColS = 0;     // score tile (128 columns)
// O_t: 144 columns, the 128 output channels and (column 128) the block row sum
// that PV accumulates against a ones row of B; the rest holds the P codes and
// the UE8M0 scale vectors (A's shared by both tiles: all 2^0; B's double-
// buffered by key-block parity: 2^e_j for the 128 channels, 2^0 for the ones rows)
constexpr uint32_t kColO0 = 128, kColO1 = 288;
constexpr uint32_t kColSFA = 272;
constexpr uint32_t kColSFB0 = 276, kColSFB1 = 496;
constexpr uint32_t kColCodes0 = 432, kColCodes1 = 464;
constexpr int kPvN = 144;

// dynamic shared memory layout (offsets from a 1024-aligned base)
constexpr uint32_t kOffQ = 0;                         // 2 x 16 KB
constexpr uint32_t kOffK = 32768;                     // kStages x 16 KB
constexpr uint32_t kVStage = 18432;                   // a V tile (16 KB) + 16 constant rows (2 KB)
constexpr uint32_t kOffV = kOffK + kStages * 16384;   // kStages x 18 KB
constexpr uint32_t kOffL = kOffV + kStages * kVStage; // 2 tiles x (hi 4 KB + lo 4 KB)
constexpr uint32_t kOffMu = kOffL + 16384;            // 2 buffers x 4 KB
constexpr uint32_t kSmemBytes = kOffMu + 8192;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;

struct AttnParams {
  CUtensorMap tmQ, tmK, tmV;
  const float* q_scale;
  const float* k_scale;
  const int8_t* v_exp;
  const uint16_t* v_mean;
  uint16_t* O;
  float* lse;
  int N, nb;
  float c_base;            // softmax_scale * log2(e)
  DevStatus* st;
  unsigned long long wait_ns;
  float skip_log2;               // Skip Softmax: log2(lambda), -inf when off
  unsigned long long* skipped;   // optional count of skipped (query tile, key block) pairs
  const float* v_chscale;        // SAGE operands: per-channel V scale [B*H][128]
};


struct __align__(8) AttnBars {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];    // S holds tile t's scores of the current block
  uint64_t s_free[2];    // tile t's warpgroup has loaded them (S may be refilled)
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t mu_full[2];
  uint64_t mu_empty[2];
  uint64_t mma_done;
};

// offset of fp32 element (row r, col k) in a K-major, no-swizzle [128 x 8] tile
__device__ __forceinline__ uint32_t tf32_tile_off(int r, int k) {
  return (uint32_t)((r >> 3) * 256 + (k >> 2) * 128 + (r & 7) * 16 + (k & 3) * 4);
}

// SKIP: Skip Softmax (BLASST) block rejection ("Accelerating Video Generation
// with GEMM Quantization, Attention Quantization and Skip Softmax Attention in
// TensorRT-LLM", section "Sparse Attention with Skip Softmax"): row i drops key
// block j when exp(block max - running max) < lambda.  Rejected rows write code
// 0 (no probability, zero row sum); a warp whose 32 rows all reject skips its
// code pass (it stores zero codes), and when all four warps of a query tile do,
// the MMA warp skips the tile's PV.
// SAGE: operands of the SAGE-style comparison recipe (vca_sage_quantize_qkv):
// one Q scale per token, one K scale per 16 keys, V with per-channel scales
// applied to the output and no block exponents or means (no mean restore).
// QI8 (SAGE only): Q and K are INT8 codes, QK^T runs as kind::i8 into s32
// accumulators, converted exactly to fp32 (|q.k| < 2^21) after the load.
// 64 consecutive 32-bit TMEM columns of this thread's lane -> registers.
#define VCA_TMEM_LD64(taddr, r)                                                                     \
  asm volatile(                                                                                     \
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15," \
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38," \
      "%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61," \
      "%62,%63}, [%64];"                                                                            \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), \
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),        \
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),      \
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),      \
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]),      \
        "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),      \
        "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),      \
        "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),      \
        "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])       \
      : "r"(taddr))

// one / four 32-bit TMEM columns of this thread's lane <- registers
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v));
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3]));
}

// block row sum l -> L tile entry (row r, block kk of the group): the hi part
// exact in TF32, lo the remainder
__device__ __forceinline__ void store_l(uint8_t* sLt, int r, int kk, float l) {
  const float hi = __uint_as_float(__float_as_uint(l) & 0xFFFFE000u);
  *reinterpret_cast<float*>(sLt + tf32_tile_off(r, kk)) = hi;
  *reinterpret_cast<float*>(sLt + 4096 + tf32_tile_off(r, kk)) = l - hi;
}

template <bool SKIP, bool SAGE, bool QI8 = false>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_fp8_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ AttnBars bars;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int never_s;   // abort flag for drain waits: these must not give up early
  // Skip Softmax: byte w of warp_drop_s[t] is 1 when warp w of tile t dropped the
  // current block (one 32-bit read tells the MMA warp whether the whole tile did)
  __shared__ uint32_t warp_drop_s[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int N = p.N, nb = p.nb, nkv = nb;
  const int ngroups = (nkv + kGroup - 1) / kGroup;
  const int64_t Np = (int64_t)nb * 128;
  const uint64_t lim = p.wait_ns;

  if (threadIdx.x == 0) {
    abort_s = 0;
    never_s = 0;
    warp_drop_s[0] = warp_drop_s[1] = 0u;
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
  // rows 128-143 of every V stage (after the 16 KB the TMA fills): row 128 all
  // E4M3 1.0, the rest zero, so PV's B operand has a row of ones and its
  // column 128 of O accumulates the row sum (the 128-byte swizzle permutes 16-byte
  // chunks within a row, which leaves a constant row as it is)
  for (int i = threadIdx.x; i < kStages * 512; i += kAttnThreads) {
    const int s = i >> 9, off = (i & 511) * 4;
    *reinterpret_cast<uint32_t*>(sm + kOffV + s * kVStage + 16384 + off) = off < 128 ? 0x38383838u : 0u;
  }
  fence_proxy_async_smem();
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
        mbar_arrive_expect_tx(&bars.kv_full[s], 32768);
        tma_load_2d(sm + kOffK + s * 16384, &p.tmK, &bars.kv_full[s], 0, (int)((int64_t)bh * Np) + j * 128);
        tma_load_2d(sm + kOffV + s * kVStage, &p.tmV, &bars.kv_full[s], j * 128, bh * 128);
        issued = j + 1;
      }
      if (abort_s) {
        // let the copies already issued land before the CTA exits
        for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
          mbar_wait_bounded(&bars.kv_full[j % kStages], (j / kStages) & 1, &never_s, nullptr, lim, 101);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in lockstep, so descriptors are computed
    // once, stay warp-uniform and advance by constants; one elected lane issues
    // the tcgen05 instructions, one election per QK^T or PV (its four K steps
    // and the commit).  (The issuing warp shares its SM sub-partition with two
    // softmax warps: the fewer instructions per MMA, the sooner the tensor pipe
    // gets its next operation.)
    const uint32_t id_qk = QI8 ? instr_desc_s8(128, 128) : instr_desc(kFmtE4M3, kFmtE4M3, 128, 128, 0, 0);
    const uint32_t id_pv = instr_desc_mx(kFmtE4M3, kFmtE4M3, 128, kPvN);
    const uint32_t id_mu = instr_desc(kFmtTF32, kFmtTF32, 128, 128, 0, 0);
    // descriptor start addresses count 16-byte units: +2 per 32-byte K step,
    // +1024 per 16 KB tile, +256 per 4 KB
    const uint64_t dQ = smem_desc(smem_u32(sm + kOffQ), 16, 1024, kLayoutSW128);
    const uint64_t dK = smem_desc(smem_u32(sm + kOffK), 16, 1024, kLayoutSW128);
    const uint64_t dV = smem_desc(smem_u32(sm + kOffV), 16, 1024, kLayoutSW128);
    const uint64_t dL = smem_desc(smem_u32(sm + kOffL), 128, 256, kLayoutNone);
    const uint64_t dMu = smem_desc(smem_u32(sm + kOffMu), 128, 256, kLayoutNone);
    unsigned long long nskip = 0;   // Skip Softmax: PVs skipped by this CTA
    const uint32_t tS = tmem + kColS;
    // S <- Q_t K_jj^T (K_jj in stage jj % kStages, already waited for)
    auto issue_qk = [&](int t, int jj) {
      const int s1 = jj % kStages;
      if (QI8)
        VCA_MMA4_SS_W("i8", tS, dQ + (uint64_t)(t * 1024), dK + (uint64_t)(s1 * 1024), id_qk, 0u, &bars.s_full[t]);
      else
        VCA_MMA4_SS_W("f8f6f4", tS, dQ + (uint64_t)(t * 1024), dK + (uint64_t)(s1 * 1024), id_qk, 0u,
                      &bars.s_full[t]);
    };
    // mean restore of group g: O_t += L_t(g) M(g) (L split hi + lo); after
    // tile 1's, the block-mean buffer may be refilled
    auto issue_mu = [&](int t, int g) -> bool {
      const int gb = g & 1;
      if (!mbar_wait_warp(&bars.mu_full[gb], (g >> 1) & 1, &abort_s, p.st, lim, 220)) return false;
      tc_fence_after();
      const uint64_t bdesc = dMu + (uint64_t)(gb * 256);
      const uint32_t tOt = tmem + (t ? kColO1 : kColO0);
      mma_tf32_ss_w(tOt, dL + (uint64_t)(t * 512), bdesc, id_mu, 1u);
      mma_tf32_ss_w(tOt, dL + (uint64_t)(t * 512 + 256), bdesc, id_mu, 1u);
      if (t == 1) tc_commit_w(&bars.mu_empty[gb]);
      return true;
    };
    // O_t += P_t(j) R_j 2^e_j, and in column 128 the block row sum P_t(j) 1 (B's
    // ones row); the L tile of a group is complete once the warpgroup has read
    // the row sums of its last block, so a group's mean restore is issued with
    // the next group's first PV (the last group's after the loop).  o_done[t]
    // then tracks everything that reads P_t or the scale vectors, or writes O_t.
    auto issue_pv = [&](int t, int j) -> bool {
      if (!mbar_wait_warp(&bars.p_full[t], j & 1, &abort_s, p.st, lim, 210 + t)) return false;
      tc_fence_after();
      const int s = j % kStages;
      const uint32_t tCodes = tmem + (t ? kColCodes1 : kColCodes0);
      const uint32_t tSFB = tmem + ((j & 1) ? kColSFB1 : kColSFB0);
      // (the flags were written before the warpgroup's p_full arrivals)
      bool skip_pv = false;
      if (SKIP) {
        skip_pv = *reinterpret_cast<const volatile uint32_t*>(&warp_drop_s[t]) == 0x01010101u;
        nskip += skip_pv ? 1 : 0;
      }
      if (!SAGE && j > 0 && j % kGroup == 0 && !issue_mu(t, j / kGroup - 1)) return false;
      if (!skip_pv)   // 8 columns (32 codes) per K step
        VCA_MMA4_MXF8_TS_W(tmem + (t ? kColO1 : kColO0), tCodes, dV + (uint64_t)(s * (kVStage / 16)), id_pv,
                           tmem + kColSFA, tSFB, j > 0 ? 1u : 0u, &bars.o_done[t]);
      else
        tc_commit_w(&bars.o_done[t]);
      return true;
    };
    // after the last block: the warpgroup has added the last row sums to the
    // L tile; the last group's mean restore completes O_t
    auto issue_last = [&](int t) -> bool {
      if (!mbar_wait_warp(&bars.p_full[t], nkv & 1, &abort_s, p.st, lim, 240 + t)) return false;
      tc_fence_after();
      if (!SAGE && !issue_mu(t, (nkv - 1) / kGroup)) return false;
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
      if (j + 1 < nkv) {   // tile 0 has loaded S_0(j+1): S takes tile 1's scores
        ok = mbar_wait_warp(&bars.s_free[0], (j + 1) & 1, &abort_s, p.st, lim, 230);
        if (!ok) break;
        tc_fence_after();
        issue_qk(1, j + 1);
      }
      ok = issue_pv(1, j);
      if (!ok) break;
      tc_commit_w(&bars.kv_empty[j % kStages]);   // K_j and V_j are no longer read
      if (j + 2 < nkv) {   // tile 1 has loaded S_1(j+1): S takes tile 0's next scores
        const int s2 = (j + 2) % kStages;
        ok = mbar_wait_warp(&bars.s_free[1], (j + 1) & 1, &abort_s, p.st, lim, 231) &&
             mbar_wait_warp(&bars.kv_full[s2], ((j + 2) / kStages) & 1, &abort_s, p.st, lim, 232);
        if (!ok) break;
        tc_fence_after();
        issue_qk(0, j + 2);
      }
    }
    ok = ok && issue_last(0);
    ok = ok && issue_last(1);
    tc_commit_w(&bars.mma_done);
    if (SKIP && lane == 0 && p.skipped && nskip) atomicAdd(p.skipped, nskip);
  } else if (warp == 2 && !SAGE) {
    // ------------------------------------------------------------ block means -> fp32 [d][8] tiles
    const uint16_t* vm = p.v_mean + (int64_t)bh * nb * 128;
    for (int g = 0; g < ngroups; ++g) {
      const int gb = g & 1, u = g >> 1;
      if (u > 0 && !mbar_wait_bounded(&bars.mu_empty[gb], (u - 1) & 1, &abort_s, p.st, lim, 300)) break;
      uint8_t* dst = sm + kOffMu + gb * 4096;
      for (int q = 0; q < 4; ++q) {
        const int dch = q * 32 + lane;
        for (int kk = 0; kk < kGroup; ++kk) {
          const int blk = g * kGroup + kk;
          float v = blk < nb ? __uint_as_float((uint32_t)__ldg(vm + (int64_t)blk * 128 + dch) << 16) : 0.0f;
          *reinterpret_cast<float*>(dst + tf32_tile_off(dch, kk)) = v;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars.mu_full[gb]);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp >> 2) - 1;                 // query tile of this warpgroup
    const int r = threadIdx.x & 127;               // query row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + kColS + lane_off;
    const uint32_t tCodes = tmem + (t ? kColCodes1 : kColCodes0) + lane_off;   // this tile's P codes
    const uint32_t tO = tmem + (t ? kColO1 : kColO0) + lane_off;
    const uint32_t tRS = tO + 128;                 // the row sum PV accumulates (read and zeroed per block)
    const int qtile = pair * 2 + t;
    const bool qvalid = qtile < nb;
    const bool row_valid = qvalid && qtile * 128 + r < N;
    const float sq = !qvalid ? 1.0f
                     : SAGE ? __ldg(p.q_scale + (int64_t)bh * Np + (int64_t)qtile * 128 + r)
                            : __ldg(p.q_scale + (int64_t)bh * nb + qtile);
    const float cq = sq * p.c_base;
    const float kMagic = 12582912.0f;              // 1.5 * 2^23: adding it rounds to an integer
    uint8_t* sLt = sm + kOffL + t * 8192;
    const float* ksc = p.k_scale + (int64_t)bh * nb;
    const int8_t* vex = p.v_exp + (int64_t)bh * nb;
    int nref = 0;
    bool have_ref = false;
    float zrun = -INFINITY;        // Skip Softmax: running maximum of the block maxima (log2 units)
    float ltot = 0.0f;
    bool ok = true;
    // the next tile's K scale and V exponent are loaded one tile ahead, off the
    // critical path of the score -> code computation
    // SAGE: eight K scales per key block (one per 16 keys)
    const float* ksc16 = p.k_scale + (int64_t)bh * (Np / 16);
    float ksc_next = SAGE ? 0.0f : __ldg(ksc);
    int vex_next = SAGE ? 0 : __ldg(vex);
    float k8_next[8];
    if (SAGE) {
#pragma unroll
      for (int g = 0; g < 8; ++g) k8_next[g] = __ldg(ksc16 + g);
    }
    for (int j = 0; j < nkv; ++j) {
      const float ksc_j = ksc_next;
      const int vex_j = vex_next;
      float k8[8];
      if (SAGE) {
#pragma unroll
        for (int g = 0; g < 8; ++g) k8[g] = k8_next[g];
      }
      if (j + 1 < nkv) {
        if (SAGE) {
#pragma unroll
          for (int g = 0; g < 8; ++g) k8_next[g] = __ldg(ksc16 + (j + 1) * 8 + g);
        } else {
          ksc_next = __ldg(ksc + j + 1);
          vex_next = __ldg(vex + j + 1);
        }
      }
      ok = mbar_wait_warp(&bars.s_full[t], j & 1, &abort_s, p.st, lim, 400 + t);
      if (!ok) break;
      tc_fence_after();
      float sv[128];
      {
        uint32_t* su = reinterpret_cast<uint32_t*>(sv);
        VCA_TMEM_LD64(tS + 0, (su + 0));
        VCA_TMEM_LD64(tS + 64, (su + 64));
        tmem_ld_wait();
      }
      // the scores are in registers: S may take the other tile's next scores
      tc_fence_before();
      mbar_arrive(&bars.s_free[t]);
      if (QI8) {
        // s32 -> fp32 exactly: the integer sits in the mantissa of 1.5 * 2^23
        uint32_t* su = reinterpret_cast<uint32_t*>(sv);
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float2 f = __fadd2_rn(make_float2(__uint_as_float(su[c] + 0x4B400000u),
                                                  __uint_as_float(su[c + 1] + 0x4B400000u)),
                                      make_float2(-kMagic, -kMagic));
          sv[c] = f.x;
          sv[c + 1] = f.y;
        }
      }
      const int valid = min(128, N - j * 128);
      if (valid < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) sv[c] = -INFINITY;
      }
      float mx = 0.0f, zmx = 0.0f;   // block maximum: raw score / in log2 units (SAGE)
      float c8g[8];                   // SAGE: code multiplier of each 16-key group
      if (!SAGE) {
        // row maximum: four independent chains of 3-input max, chain q over the
        // 32 scores sv[32q .. 32q+31]
        float mq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float m = sv[32 * q];
#pragma unroll
          for (int i = 1; i < 31; i += 2) m = fmax3(m, sv[32 * q + i], sv[32 * q + i + 1]);
          mq[q] = fmaxf(m, sv[32 * q + 31]);
        }
        mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
      } else {
        // one chain per 16-key group (its own K scale): z max = max_g(max s * cz_g)
        zmx = -INFINITY;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float m = sv[16 * g];
#pragma unroll
          for (int i = 1; i < 15; i += 2) m = fmax3(m, sv[16 * g + i], sv[16 * g + i + 1]);
          m = fmaxf(m, sv[16 * g + 15]);
          const float czg = cq * k8[g];
          c8g[g] = 8.0f * czg;
          zmx = fmaxf(zmx, m * czg);
        }
      }
      const float cz = cq * ksc_j;                 // z = s * cz (log2 domain)
      const float c8 = 8.0f * cz;
      bool rej = false;           // Skip Softmax: this row drops the block
      if (SKIP) {
        const float zt = SAGE ? zmx : mx * cz;
        zrun = fmaxf(zrun, zt);
        // rows past the end of the sequence (padding of the last query tile)
        // vote to drop every block, so they never hold a whole-tile skip back
        rej = j > 0 && (!row_valid || zt - zrun < p.skip_log2);
      }
      const int ntile = (int)ceilf(SAGE ? zmx - 0.08125f : __fmaf_rn(mx, cz, -0.08125f));
      float rescale = 1.0f;       // O_t and the pending row sums are scaled by this
      if (rej) {
        // a dropped block lies below the running maximum, which the reference
        // trails by at most 4 octaves: it leaves the reference where it is
      } else if (!have_ref) {
        nref = ntile;
        have_ref = true;
      } else if (ntile > nref + 4) {
        const int delta = ntile - nref;
        nref = ntile;
        rescale = delta > 126 ? 0.0f : __uint_as_float((uint32_t)(127 - delta) << 23);
      }
      // ExpCast: code = rne(s*c8 + 87 - 8*nref) via the magic-number FMA (two
      // scores per fma.rn.f32x2), clamped below at 0; the block's row sum of the
      // decoded probabilities comes from the tensor core (PV's row of ones, in
      // column 128 of O_t), read one block later
      const bool warp_drop = SKIP && __all_sync(0xffffffffu, rej);
      // a dropped row writes code 0 everywhere: multiplier 0, addend the bare magic constant
      const float badd = rej ? kMagic : kMagic + (float)(87 - 8 * nref);
      const float c8r = rej ? 0.0f : c8;
      const float2 c8x2 = make_float2(c8r, c8r), baddx2 = make_float2(badd, badd);
      uint32_t pw[32];   // the row's 128 codes, 4 per word, in key order
      // PV_t(j-1), its row sums (and any mean restore before it) must have
      // completed before the P region, sL_t or O_t are written; they were
      // issued when this warpgroup finished the previous block, so this wait
      // rarely blocks.  The row sum of block j-1 is loaded here and used after
      // the code pass.
      uint32_t lprev_bits = 0;
      if (j > 0) {
        ok = mbar_wait_warp(&bars.o_done[t], (j - 1) & 1, &abort_s, p.st, lim, 410 + t);
        if (!ok) break;
        tc_fence_after();
        lprev_bits = tmem_ld1(tRS);
      }
      if (warp_drop) {
        // PV may still run for the other warps' rows: these rows contribute zeros
        const uint32_t zero[32] = {};
        VCA_TMEM_ST32(tCodes, zero);
      } else {
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const int c = q * 4;
        const float c8q = SAGE ? (rej ? 0.0f : c8g[q >> 2]) : 0.0f;
        const float2 cx = SAGE ? make_float2(c8q, c8q) : c8x2;
        const float2 f01 = __ffma2_rn(make_float2(sv[c], sv[c + 1]), cx, baddx2);
        const float2 f23 = __ffma2_rn(make_float2(sv[c + 2], sv[c + 3]), cx, baddx2);
        const uint32_t b0 = __float_as_uint(fmaxf(f01.x, kMagic)), b1 = __float_as_uint(fmaxf(f01.y, kMagic));
        const uint32_t b2 = __float_as_uint(fmaxf(f23.x, kMagic)), b3 = __float_as_uint(fmaxf(f23.y, kMagic));
        pw[q] = prmt(prmt(b0, b1, 0x0040u), prmt(b2, b3, 0x0040u), 0x5410u);
      }
      VCA_TMEM_ST32(tCodes, pw);
      }
      if (j > 0) {
        // block j-1's row sum (in the units of the reference before this
        // block's rescale) -> L tile and the running total
        tmem_ld_wait();
        reg_after_wait(lprev_bits);
        tmem_st1(tRS, 0u);   // the next PV adds block j's row sum to zero
        const float lprev = __uint_as_float(lprev_bits);   // sum of the E4M3 values
        if (!SAGE) store_l(sLt, r, (j - 1) % kGroup, lprev);
        ltot += lprev;
      }
      // tcgen05.ld/st are warp-collective: if any row of the warp rescales, the
      // whole warp runs the read-modify-write (other rows multiply by 1)
      if (__any_sync(0xffffffffu, rescale != 1.0f)) {
        // the reference maximum moved up: O_t and this group's earlier row sums
        // are scaled by the same exact power of two (S is no longer live here)
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t o[32];
          VCA_TMEM_LD32(tO + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * rescale);
          VCA_TMEM_ST32(tO + c0, o);
        }
        // the L entries not yet restored: those of block j-1's group
        for (int kk = 0; kk <= (SAGE ? -1 : (j - 1) % kGroup); ++kk) {
          float* hi = reinterpret_cast<float*>(sLt + tf32_tile_off(r, kk));
          float* lo = reinterpret_cast<float*>(sLt + 4096 + tf32_tile_off(r, kk));
          *hi *= rescale;
          *lo *= rescale;
        }
      }
      ltot *= rescale;
      // UE8M0 scale vectors, written by tile 0's warpgroup (the PV of tile 1 for
      // the same key block comes after tile 0's): A = 2^0 (once), B = 2^v_exp[j]
      // for the 128 channel rows and 2^0 for the ones rows (fifth column)
      if (t == 0) {
        if (j == 0) {
          const uint32_t one4[4] = {0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu};
          tmem_st4(tmem + kColSFA + lane_off, one4);
        }
        const uint32_t eb = (uint32_t)(127 + vex_j) * 0x01010101u;
        const uint32_t sf[8] = {eb, eb, eb, eb, 0x7F7F7F7Fu, 0u, 0u, 0u};
        tmem_st8(tmem + ((j & 1) ? kColSFB1 : kColSFB0) + lane_off, sf);
      }
      if (SKIP && lane == 0) reinterpret_cast<volatile uint8_t*>(&warp_drop_s[t])[warp & 3] = warp_drop ? 1 : 0;
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars.p_full[t]);
    }
    // ------------------------------------------------------------ last row sums
    // the last block's row sum completes the L tile (zero past the last block)
    // and the total; the MMA warp then issues the last group's mean restore
    if (ok) ok = mbar_wait_warp(&bars.o_done[t], (nkv - 1) & 1, &abort_s, p.st, lim, 420 + t);
    if (ok) {
      tc_fence_after();
      uint32_t lb = tmem_ld1(tRS);
      tmem_ld_wait();
      reg_after_wait(lb);
      const float llast = __uint_as_float(lb);
      ltot += llast;
      if (!SAGE) {
        const int kk = (nkv - 1) % kGroup;
        store_l(sLt, r, kk, llast);
        for (int k2 = kk + 1; k2 < kGroup; ++k2) store_l(sLt, r, k2, 0.0f);
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(&bars.p_full[t]);
      ok = mbar_wait_warp(&bars.o_done[t], nkv & 1, &abort_s, p.st, lim, 430 + t);
    }
    // ------------------------------------------------------------ epilogue
    if (ok) {
      tc_fence_after();
      const int qrow = qtile * 128 + r;
      const bool store = qvalid && qrow < N;
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
            float o0 = __uint_as_float(o[2 * c]) * inv, o1 = __uint_as_float(o[2 * c + 1]) * inv;
            if (SAGE) {
              o0 *= __ldg(p.v_chscale + bh * 128 + c0 + 2 * c);
              o1 *= __ldg(p.v_chscale + bh * 128 + c0 + 2 * c + 1);
            }
            __nv_bfloat162 h = __floats2bfloat162_rn(o0, o1);
            pk[c] = *reinterpret_cast<uint32_t*>(&h);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      if (store && p.lse)
        p.lse[(int64_t)bh * N + qrow] = 0.69314718055994531f * ((float)nref + 0.08125f - 4.0f + __log2f(ltot));
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every issued MMA has completed before TMEM is released
    mbar_wait_bounded(&bars.mma_done, 0, &never_s, nullptr, lim, 500);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace vca

using namespace vca;

extern "C" size_t vca_attention_workspace_size(int B, int H, int N) { return 256; }

static int attention_launch(const char* fn, const void* Qq, const float* q_scale, const void* Kq,
                            const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                            const vca_bf16* v_mean, int B, int H, int N, int d, float softmax_scale,
                            vca_bf16* O, float* lse, void* ws, size_t ws_bytes, float skip_lambda,
                            unsigned long long* skipped, const float* v_chscale, vca_stream_t stream,
                            bool qk_i8 = false) {
  const bool sage = v_chscale != nullptr;   // SAGE operands: no V exponents or means
  if (d != VCA_HEAD_DIM) return fail(VCA_ERR_UNSUPPORTED, "%s: d must be 128", fn);
  if (B < 1 || H < 1 || N < 1 || (int64_t)B * H > 65535)
    return fail(VCA_ERR_INVALID, "%s: bad shape B=%d H=%d N=%d", fn, B, H, N);
  const int nb = (N + 127) / 128;
  const int64_t Np = (int64_t)nb * 128;
  if ((int64_t)B * H * Np > INT32_MAX || Np > INT32_MAX / 2)
    return fail(VCA_ERR_UNSUPPORTED, "%s: B*H*Np exceeds the 2^31 row limit", fn);
  const void* ptrs[] = {Qq, q_scale, Kq, k_scale, VrT, O};
  for (const void* q : ptrs)
    if (!q) return fail(VCA_ERR_INVALID, "%s: null pointer", fn);
  if (!sage && (!v_exp || !v_mean)) return fail(VCA_ERR_INVALID, "%s: null pointer", fn);
  const void* al[] = {Qq, Kq, VrT, O};
  for (const void* q : al)
    if (!aligned16(q)) return fail(VCA_ERR_INVALID, "%s: tensors must be 16-byte aligned", fn);
  if (!(softmax_scale > 0.0f)) return fail(VCA_ERR_INVALID, "%s: softmax_scale must be > 0", fn);
  if (!(skip_lambda >= 0.0f && skip_lambda < 1.0f))
    return fail(VCA_ERR_INVALID, "%s: skip_lambda must be in [0, 1)", fn);
  if (!ws || ws_bytes < vca_attention_workspace_size(B, H, N))
    return fail(VCA_ERR_WORKSPACE, "%s: workspace too small", fn);

  AttnParams prm;
  const uint64_t BH = (uint64_t)B * H;
  {
    uint64_t dims[2] = {128, BH * (uint64_t)Np}, str[1] = {128};
    uint32_t box[2] = {128, 128};
    int rc = encode_tiled(&prm.tmQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, Qq, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!rc) rc = encode_tiled(&prm.tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, Kq, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    uint64_t vd[2] = {(uint64_t)Np, BH * 128}, vs[1] = {(uint64_t)Np};
    if (!rc) rc = encode_tiled(&prm.tmV, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, VrT, vd, vs, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  prm.q_scale = q_scale;
  prm.k_scale = k_scale;
  prm.v_exp = v_exp;
  prm.v_mean = v_mean;
  prm.O = O;
  prm.lse = lse;
  prm.N = N;
  prm.nb = nb;
  prm.c_base = (float)((double)softmax_scale * 1.4426950408889634);
  prm.st = (DevStatus*)ws;
  prm.wait_ns = wait_limit_ns();
  const bool skip = skip_lambda > 0.0f;
  prm.skip_log2 = skip ? (float)log2((double)skip_lambda) : -INFINITY;
  prm.skipped = skipped;
  prm.v_chscale = v_chscale;
  if (skip && sage) return fail(VCA_ERR_UNSUPPORTED, "%s: Skip Softmax on SAGE operands is not built", fn);
  if (qk_i8 && !sage) return fail(VCA_ERR_UNSUPPORTED, "%s: INT8 QK^T is built for SAGE operands only", fn);
  auto kern = skip    ? attn_fp8_kernel<true, false>
              : qk_i8 ? attn_fp8_kernel<false, true, true>
              : sage  ? attn_fp8_kernel<false, true>
                      : attn_fp8_kernel<false, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc) != cudaSuccess)
    return fail(VCA_ERR_CUDA, "%s: cannot set shared-memory size", fn);
  dim3 grid((nb + 1) / 2, (unsigned)BH);
  kern<<<grid, kAttnThreads, kSmemAlloc, (cudaStream_t)stream>>>(prm);
  return check_launch("attn_fp8_kernel");
}

extern "C" int vca_attention_fwd(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                                 const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                                 const vca_bf16* v_mean, int B, int H, int N, int d,
                                 float softmax_scale, vca_bf16* O, float* lse, void* ws,
                                 size_t ws_bytes, vca_stream_t stream) {
  return attention_launch("vca_attention_fwd", Qq, q_scale, Kq, k_scale, VrT, v_exp, v_mean, B, H, N, d,
                          softmax_scale, O, lse, ws, ws_bytes, 0.0f, nullptr, nullptr, stream);
}

extern "C" int vca_attention_fwd_skip(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                                      const float* k_scale, const uint8_t* VrT, const int8_t* v_exp,
                                      const vca_bf16* v_mean, int B, int H, int N, int d,
                                      float softmax_scale, float skip_lambda, vca_bf16* O, float* lse,
                                      unsigned long long* skipped_tiles, void* ws, size_t ws_bytes,
                                      vca_stream_t stream) {
  return attention_launch("vca_attention_fwd_skip", Qq, q_scale, Kq, k_scale, VrT, v_exp, v_mean, B, H, N, d,
                          softmax_scale, O, lse, ws, ws_bytes, skip_lambda, skipped_tiles, nullptr, stream);
}

extern "C" int vca_attention_fwd_sage(const uint8_t* Qq, const float* q_scale, const uint8_t* Kq,
                                      const float* k_scale, const uint8_t* VcT, const float* v_chscale, int B,
                                      int H, int N, int d, float softmax_scale, vca_bf16* O, float* lse, void* ws,
                                      size_t ws_bytes, vca_stream_t stream) {
  if (!v_chscale) return fail(VCA_ERR_INVALID, "vca_attention_fwd_sage: null pointer");
  return attention_launch("vca_attention_fwd_sage", Qq, q_scale, Kq, k_scale, VcT, nullptr, nullptr, B, H, N, d,
                          softmax_scale, O, lse, ws, ws_bytes, 0.0f, nullptr, v_chscale, stream);
}

extern "C" int vca_attention_fwd_sage_i8(const int8_t* Qq, const float* q_scale, const int8_t* Kq,
                                         const float* k_scale, const uint8_t* VcT, const float* v_chscale, int B,
                                         int H, int N, int d, float softmax_scale, vca_bf16* O, float* lse,
                                         void* ws, size_t ws_bytes, vca_stream_t stream) {
  if (!v_chscale) return fail(VCA_ERR_INVALID, "vca_attention_fwd_sage_i8: null pointer");
  return attention_launch("vca_attention_fwd_sage_i8", Qq, q_scale, Kq, k_scale, VcT, nullptr, nullptr, B, H, N,
                          d, softmax_scale, O, lse, ws, ws_bytes, 0.0f, nullptr, v_chscale, stream, true);
}
