// vca_kmeans.cu -- V-Smooth grouping: k-means over value tokens and the stable
// permutation that sorts tokens by cluster.
//
// Method: "VC-Attention: Training-Free Low-Bit Attention Speeds Video Diffusion
// Up to 3.6x" (V-Smooth bullet): value tokens are reordered by lightweight
// online clustering so a hardware block holds tokens that quantise well
// together; "VC-Attention" (aikraft.ru, section "Решение"): a lightweight
// k-means groups similar tokens into blocks; "Nunchux AI Introduces
// VC-Attention..." (abstract): the block mean removes far more energy after
// sorting.
//
// Per round: assign (token-parallel; fp32 distances in channel order, one FMA
// per channel, so the argmin is reproducible bit for bit; a tensor-core
// estimate with a proven error bound picks the centroids whose distance is
// evaluated), accumulate
// (channel-parallel exact 2^-24 fixed-point sums in int64, order-free), update
// (one fp64 division per centroid coordinate).  Then a stable counting sort:
// per-chunk histograms, an exclusive scan in (cluster, chunk) order, and a
// warp-synchronous ranked scatter.
#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

constexpr int kSortChunk = 1024;    // tokens per sort CTA

struct KmWs {
  DevStatus* st;
  long long* sums;   // [BH][k][128]
  int* counts;       // [BH][k]
  int* ccount;       // [BH][nchunk][k]  per-chunk histogram
  int* cbase;        // [BH][nchunk][k]  scatter base per (chunk, cluster)
  int* cstart;       // [BH][k]          first sorted position of each cluster
};

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static KmWs carve(void* ws, int BH, int N, int k, size_t* total) {
  size_t nchunk = (size_t)(N + kSortChunk - 1) / kSortChunk;
  size_t off = 0;
  KmWs w;
  char* base = (char*)ws;
  w.st = (DevStatus*)(base + off);
  off += 256;
  w.sums = (long long*)(base + off);
  off += align256((size_t)BH * k * 128 * sizeof(long long));
  w.counts = (int*)(base + off);
  off += align256((size_t)BH * k * sizeof(int));
  w.ccount = (int*)(base + off);
  off += align256((size_t)BH * nchunk * k * sizeof(int));
  w.cbase = (int*)(base + off);
  off += align256((size_t)BH * nchunk * k * sizeof(int));
  w.cstart = (int*)(base + off);
  off += align256((size_t)BH * k * sizeof(int));
  *total = off;
  return w;
}

// centroid c of head bh = token floor(c*N/k), or the caller's warm start
__global__ void km_init_kernel(const uint16_t* __restrict__ V, const float* __restrict__ init,
                               float* __restrict__ cent, int N, int k) {
  int bh = blockIdx.x, c = blockIdx.y, ch = threadIdx.x;
  float* dst = cent + ((int64_t)bh * k + c) * 128;
  if (init) {
    dst[ch] = init[((int64_t)bh * k + c) * 128 + ch];
  } else {
    int64_t src = ((int64_t)c * N) / k;
    dst[ch] = __uint_as_float((uint32_t)V[((int64_t)bh * N + src) * 128 + ch] << 16);
  }
}

// ---------------------------------------------------------------- assignment
// The assignment keeps the distance's defined arithmetic -- for centroid mu,
// t_i = v_i - mu_i rounded to fp32 and D = fma(t_i, t_i, D) over the channels
// in order 0..127 from D = 0, the lowest index winning ties -- but evaluates it
// only for the centroids that can win.  A tensor-core estimate
//   d_c = |v|^2 + |mu_c|^2 - 2 v.mu_c
// (v.mu_c from the bf16 V tile against the centroids split into bf16 hi + lo,
// both accumulated in fp32 in tensor memory) differs from the defined D_c by less
// than e_c = 2^-10 (|v|^2 + |mu_c|^2) + 2^-90:
//  * the split leaves at most 2^-18 |mu_i| per coordinate, the bf16 products
//    are exact, and the fp32 sums of at most 256 products err by less than
//    2^-14 of their absolute sum, which is at most (|v|^2 + |mu|^2) / 2;
//  * |v|^2 and |mu|^2 are fp32 sums of 128 exact squares (error below 2^-17
//    of each), and the last two operations round once each;
//  * D_c itself is within 131 units of 2^-24 of the exact squared distance,
//    which is at most 2 (|v|^2 + |mu|^2);
// together below 10^-4 of |v|^2 + |mu_c|^2, a tenth of the margin, and the
// absolute term covers subnormal flushing.  Every centroid whose D_c is the
// minimum therefore satisfies d_c - e_c <= min_k (d_k + e_k); the exact D is
// computed for those candidates only, in increasing index, which gives the
// full scan's result bit for bit.  A non-finite estimate anywhere sends the
// token through all k centroids in the defined way.
constexpr int kAsgThreads = 128;              // one token per thread = TMEM lane
constexpr float kFilterRel = 0x1p-10f, kFilterAbs = 0x1p-90f;

struct AsgParams {
  CUtensorMap tmV;     // V as [BH][N][128] bf16; box 64 channels x 128 tokens, 128-byte swizzle
  const float* cent;   // [BH][k][128]
  int32_t* assign;     // [BH][N]
  DevStatus* st;
  uint64_t lim;
  int N, k;
};

// KP centroid slots (32 for k <= 32, else 64): two B matrices of KP rows, the
// bf16 hi parts and the lo parts of the centroids, accumulated into the same
// KP tensor-memory columns (column c = v.hi_c + v.lo_c, 256 products).
// Persistent over one head: CTA x takes the head's 128-token tiles x, x + G,
// x + 2G, ... (G = gridDim.x), so the centroid operand and the tensor memory are
// set up once per CTA; each thread keeps its token's row in registers, so the
// one V buffer takes the next tile's TMA copy while this tile is filtered and
// its candidates evaluated.
template <int KP>
__global__ void __launch_bounds__(kAsgThreads, 3) km_assign_kernel(const __grid_constant__ AsgParams p) {
  constexpr uint32_t kBChunk = KP * 128;   // bytes of one 64-channel chunk of a B matrix
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sV = sm;           // the token tile: 2 chunks of 64 channels x 128 rows of 128 bytes
  uint8_t* sB = sm + 32768;   // hi then lo, each 2 chunks of KP rows
  __shared__ __align__(8) uint64_t bar_full, bar_mma;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s, never_s;
  __shared__ float nc_s[KP];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.y, k = p.k, G = gridDim.x;
  const int ntiles = (p.N + 127) / 128;
  if (tid == 0) {
    abort_s = 0;
    never_s = 0;
    mbar_init(&bar_full, 1);
    mbar_init(&bar_mma, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(&bar_full, 32768);   // the first tile (blockIdx.x < ntiles)
    tma_load_3d(sV, &p.tmV, &bar_full, 0, blockIdx.x * 128, bh);
    tma_load_3d(sV + 16384, &p.tmV, &bar_full, 64, blockIdx.x * 128, bh);
  }
  // B: thread pair (c, half) writes centroid c's channels 64 half .. +63 as bf16
  // hi and lo (row c of either matrix) in 16-byte units swizzled by the row
  // index (the layout of a 128-byte-swizzle TMA box) and sums |mu_c|^2
  {
    const int c = tid >> 1, half = tid & 1;
    if (c < KP) {   // warp-uniform: a warp holds 16 consecutive c
      const float4* src = reinterpret_cast<const float4*>(p.cent + ((int64_t)bh * k + (c < k ? c : 0)) * 128) +
                          half * 16;
      uint8_t* hrow = sB + half * kBChunk + c * 128;
      uint8_t* lrow = sB + (2 + half) * kBChunk + c * 128;
      float ss = 0.0f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {   // channels 64 half + 8u .. +7
        float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f), b = a;
        if (c < k) {
          a = __ldg(src + 2 * u);
          b = __ldg(src + 2 * u + 1);
        }
        const float m[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(m[2 * e]), h1 = __float2bfloat16_rn(m[2 * e + 1]);
          const __nv_bfloat16 l0 = __float2bfloat16_rn(m[2 * e] - __bfloat162float(h0));
          const __nv_bfloat16 l1 = __float2bfloat16_rn(m[2 * e + 1] - __bfloat162float(h1));
          hw[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
          lw[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
          ss = fmaf(m[2 * e], m[2 * e], ss);
          ss = fmaf(m[2 * e + 1], m[2 * e + 1], ss);
        }
        const int su = (u ^ (c & 7)) << 4;
        *reinterpret_cast<uint4*>(hrow + su) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(lrow + su) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      if (half == 0) nc_s[c] = ss;
    }
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_s, KP);
    tmem_relinquish();
  }
  fence_proxy_async_smem();   // B's rows, written by these threads, for the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  const uint32_t idesc = instr_desc(kFmtBF16, kFmtBF16, 128, KP, 0, 0);
  const uint64_t dA = smem_desc(smem_u32(sV), 16, 1024, kLayoutSW128);
  const uint64_t dB = smem_desc(smem_u32(sB), 16, 1024, kLayoutSW128);
  const float4* cb = reinterpret_cast<const float4*>(p.cent + (int64_t)bh * k * 128);
  // for the exit after a failed wait: what may still be in flight
  bool full_ok = true, mma_issued = false, mma_ok = true;
  uint32_t ph = 0;
  for (int i = 0, tile = blockIdx.x; tile < ntiles; ++i, tile += G) {
    ph = (uint32_t)i & 1u;
    full_ok = mbar_wait_warp(&bar_full, ph, &abort_s, p.st, p.lim, 500);
    mma_issued = false;
    if (warp == 0 && full_ok) {
      // D[token][c] = sum over the 128 channels of v (hi_c + lo_c): 8 steps of 16
      // channels against each matrix
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 16; ++s) {   // +32 bytes per step inside a 128-byte row, then the next chunk
        const int st = s & 7;
        mma_bf16_ss_w(tmem, dA + (uint64_t)((st >> 2) * 1024 + (st & 3) * 2),
                      dB + (uint64_t)(((s >> 3) * 2 + (st >> 2)) * (kBChunk / 16) + (st & 3) * 2), idesc, s > 0);
      }
      tc_commit_w(&bar_mma);
      mma_issued = true;
    }
    // this thread's token: row tid of the tile (16-byte units swizzled by the
    // row index) into registers, and |v|^2
    uint32_t vr[64];
    float nv = 0.0f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      uint4 x = make_uint4(0u, 0u, 0u, 0u);
      if (full_ok)
        x = *reinterpret_cast<const uint4*>(sV + (u >> 3) * 16384 + tid * 128 + (((u & 7) ^ (tid & 7)) << 4));
      vr[4 * u] = x.x;
      vr[4 * u + 1] = x.y;
      vr[4 * u + 2] = x.z;
      vr[4 * u + 3] = x.w;
    }
#pragma unroll
    for (int w = 0; w < 64; ++w) {
      nv = fmaf(bf16_lo(vr[w]), bf16_lo(vr[w]), nv);
      nv = fmaf(bf16_hi(vr[w]), bf16_hi(vr[w]), nv);
    }
    mma_ok = full_ok && mbar_wait_warp(&bar_mma, ph, &abort_s, p.st, p.lim, 502);
    // every row is in registers and the MMA has read the tile: the buffer may
    // take the next tile (a failed wait anywhere stops every thread here)
    if (__syncthreads_or(!mma_ok)) break;
    tc_fence_after();
    if (tid == 0 && tile + G < ntiles) {
      mbar_arrive_expect_tx(&bar_full, 32768);
      tma_load_3d(sV, &p.tmV, &bar_full, 0, (tile + G) * 128, bh);
      tma_load_3d(sV + 16384, &p.tmV, &bar_full, 64, (tile + G) * 128, bh);
    }
    // pass 1: the smallest upper bound; pass 2: the candidates
    float best_ub = INFINITY;
    bool bad = !(fabsf(nv) < INFINITY);
    uint64_t cand = 0;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
#pragma unroll 1
      for (int g = 0; g < KP / 32; ++g) {
        uint32_t dv[32];
        VCA_TMEM_LD32(trow + 32 * g, dv);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c = 32 * g + j;
          if (c < k) {
            const float dot = __uint_as_float(dv[j]);
            const float sn = nv + nc_s[c];
            const float d = fmaf(-2.0f, dot, sn);
            const float e = fmaf(kFilterRel, sn, kFilterAbs);
            if (pass == 0) {
              best_ub = fminf(best_ub, d + e);
              bad = bad || !(fabsf(d) < INFINITY);
            } else if (d - e <= best_ub) {
              cand |= 1ull << c;
            }
          }
        }
      }
    }
    // every thread has read its row of D: the next tile's MMA may overwrite it
    tc_fence_before();
    __syncthreads();
    if (bad || !(best_ub < INFINITY)) cand = k == 64 ? ~0ull : (1ull << k) - 1;
    // the defined distance for the candidates, in increasing index
    int best = 0;
    float bd = 0.0f;
    bool first = true;
    while (cand) {
      const int c = __ffsll((long long)cand) - 1;
      cand &= cand - 1;
      const float4* mu = cb + c * 32;
      float acc = 0.0f;
#pragma unroll
      for (int q = 0; q < 32; ++q) {   // channels 4q .. 4q + 3
        const float4 m = __ldg(mu + q);
        float t = __fsub_rn(bf16_lo(vr[2 * q]), m.x);
        acc = __fmaf_rn(t, t, acc);
        t = __fsub_rn(bf16_hi(vr[2 * q]), m.y);
        acc = __fmaf_rn(t, t, acc);
        t = __fsub_rn(bf16_lo(vr[2 * q + 1]), m.z);
        acc = __fmaf_rn(t, t, acc);
        t = __fsub_rn(bf16_hi(vr[2 * q + 1]), m.w);
        acc = __fmaf_rn(t, t, acc);
      }
      if (first || acc < bd) {
        bd = acc;
        best = c;
        first = false;
      }
    }
    const int n = tile * 128 + tid;
    if (n < p.N) p.assign[(int64_t)bh * p.N + n] = best;
  }
  // after a failed wait, nothing may still be in flight into this CTA's memory
  if (tid == 0 && !full_ok) mbar_wait_bounded(&bar_full, ph, &never_s, nullptr, p.lim, 503);
  if (warp == 0 && mma_issued && !mma_ok) mbar_wait_warp(&bar_mma, ph, &never_s, nullptr, p.lim, 504);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, KP);
  }
}

// Exact fixed-point sums per (cluster, channel), walking the tokens in sorted
// (cluster-contiguous) order.  Each warp takes kSegTok consecutive sorted
// positions, lane l holding channels 4l .. 4l + 3 (a whole 256-byte row per
// warp load, eight rows in flight).  llrint(v * 2^24) (|v| < 2^20, at most 45
// bits) is split exactly into hi * 2^22 + lo with |hi| < 2^22, |lo| <= 2^21 by
// float operations only: hi = rne(4 v) (exact product, one rounding through
// the magic-number add), r = v - hi / 4 (exact), lo = rne(r * 2^24) (the only
// other rounding, the same as llrint's since hi * 2^22 is an integer).  The
// magic-biased bit patterns are summed in 32-bit registers and the bias is
// taken off per token at each flush (at most kSegTok < 512 terms, so the true
// sums stay below 2^31 and wrap-around is harmless); one int64 atomic per
// channel is flushed whenever the walk leaves a cluster.  Integer addition is
// exact and order-free: the sums are exact whatever the order.
constexpr int kSegTok = 256;   // sorted positions per warp
constexpr int kSegWarps = 8;
// Per 16-bit half, the larger of two unsigned values.
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__global__ void __launch_bounds__(kSegWarps * 32) km_accum_kernel(const uint16_t* __restrict__ V,
                                                                 const int32_t* __restrict__ perm,
                                                                 const int* __restrict__ cstart,
                                                                 const int* __restrict__ counts,
                                                                 long long* __restrict__ sums, int N, int k,
                                                                 DevStatus* st) {
  __shared__ int cs[VCA_MAX_CLUSTERS], ce[VCA_MAX_CLUSTERS];
  const int bh = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < k) {
    cs[threadIdx.x] = cstart[(int64_t)bh * k + threadIdx.x];
    ce[threadIdx.x] = cs[threadIdx.x] + counts[(int64_t)bh * k + threadIdx.x];
  }
  __syncthreads();
  const int q0 = (blockIdx.x * kSegWarps + warp) * kSegTok;
  if (q0 >= N) return;
  const int q1 = min(N, q0 + kSegTok);
  // the cluster holding sorted position q0 (exactly one non-empty range contains it)
  int found = -1;
  for (int c2 = lane; c2 < k; c2 += 32)
    if (cs[c2] <= q0 && q0 < ce[c2]) found = c2;
  int c = max(__reduce_max_sync(0xffffffffu, found), 0);
  int cend = ce[c];
  const uint16_t* vb = V + (int64_t)bh * N * 128;
  const int32_t* pb = perm + (int64_t)bh * N;
  unsigned long long* sb = reinterpret_cast<unsigned long long*>(sums + (int64_t)bh * k * 128);
  // lane = channels 4 lane .. 4 lane + 3 (one 8-byte load per row); exact
  // llrint(v 2^24) = hi 2^22 + lo per value, two values per fma.rn.f32x2, summed
  // as the raw bits magic + hi / magic + lo and corrected by the token count at
  // each flush (wrap-around arithmetic; |sum| < 2^31 over <= 256 tokens)
  const float kMagic = 12582912.0f;   // 1.5 * 2^23
  uint32_t hs[4] = {0u, 0u, 0u, 0u}, ls[4] = {0u, 0u, 0u, 0u};
  uint32_t ntok = 0;
  uint32_t mag2 = 0;   // largest |v| bit patterns seen (two halves): the exact sums need |v| < 2^20
  auto flush = [&]() {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int h = (int)(hs[j] - ntok * 0x4B400000u), l = (int)(ls[j] - ntok * 0x4B400000u);
      const long long v = ((long long)h << 22) + (long long)l;
      if (v != 0) atomicAdd(sb + c * 128 + 4 * lane + j, (unsigned long long)v);
      hs[j] = 0u;
      ls[j] = 0u;
    }
    ntok = 0;
  };
  for (int base = q0; base < q1; base += 32) {
    const int cnt = min(32, q1 - base);
    const int myn = lane < cnt ? __ldg(pb + base + lane) : 0;
    for (int i = 0; i < cnt; i += 8) {
      // eight tokens' rows in flight at once, each a 256-byte row per warp load
      uint2 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int n = __shfl_sync(0xffffffffu, myn, (i + u) & 31);
        x[u] = i + u < cnt ? __ldg(reinterpret_cast<const uint2*>(vb + (int64_t)n * 128) + lane) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (i + u >= cnt) break;
        const int q = base + i + u;
        if (q >= cend) {   // the walk enters the next non-empty cluster
          flush();
          do {
            ++c;
          } while (c < k - 1 && ce[c] == cs[c]);
          cend = ce[c];
        }
        mag2 = vmax_u16x2(mag2, x[u].x & 0x7FFF7FFFu);
        mag2 = vmax_u16x2(mag2, x[u].y & 0x7FFF7FFFu);
        const uint32_t wv[2] = {x[u].x, x[u].y};
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const float2 v = make_float2(__uint_as_float(wv[p] << 16), __uint_as_float(wv[p] & 0xFFFF0000u));
          // hm = magic + rne(4 v); r = v - hi / 4 (exact); lm = magic + rne(r 2^24)
          const float2 hm = __ffma2_rn(v, make_float2(4.0f, 4.0f), make_float2(kMagic, kMagic));
          const float2 hf = __fadd2_rn(hm, make_float2(-kMagic, -kMagic));
          const float2 rr = __ffma2_rn(hf, make_float2(-0.25f, -0.25f), v);
          const float2 lm = __ffma2_rn(rr, make_float2(16777216.0f, 16777216.0f), make_float2(kMagic, kMagic));
          hs[2 * p] += __float_as_uint(hm.x);
          hs[2 * p + 1] += __float_as_uint(hm.y);
          ls[2 * p] += __float_as_uint(lm.x);
          ls[2 * p + 1] += __float_as_uint(lm.y);
        }
        ++ntok;
      }
    }
  }
  flush();
  // bf16 exponent field >= 127 + 20: |v| >= 2^20 (all ones: inf or NaN)
  const uint32_t magbits = __reduce_max_sync(0xffffffffu, max(mag2 & 0xFFFFu, mag2 >> 16));
  if (lane == 0 && magbits >= 0x4980u)
    report(st, magbits >= 0x7F80u ? VCA_ERR_NONFINITE : VCA_ERR_INVALID, 600, bh);
}

__global__ void km_update_kernel(const long long* __restrict__ sums, const int* __restrict__ counts,
                                 float* __restrict__ cent, int k) {
  int bh = blockIdx.x, c = blockIdx.y, ch = threadIdx.x;
  int n = counts[(int64_t)bh * k + c];
  if (n == 0) return;   // empty cluster keeps its centroid
  long long s = sums[((int64_t)bh * k + c) * 128 + ch];
  double m = __ddiv_rn((double)s, (double)n * 16777216.0);
  cent[((int64_t)bh * k + c) * 128 + ch] = __double2float_rn(m);
}

// ---- stable counting sort by cluster
__global__ void sort_count_kernel(const int32_t* __restrict__ assign, int* __restrict__ ccount,
                                  int N, int k, int nchunk) {
  __shared__ int h[VCA_MAX_CLUSTERS];
  const int bh = blockIdx.y, chunk = blockIdx.x;
  if (threadIdx.x < k) h[threadIdx.x] = 0;
  __syncthreads();
  const int n0 = chunk * kSortChunk, n1 = min(N, n0 + kSortChunk);
  for (int n = n0 + threadIdx.x; n < n1; n += blockDim.x) atomicAdd(&h[assign[(int64_t)bh * N + n]], 1);
  __syncthreads();
  if (threadIdx.x < k) ccount[((int64_t)bh * nchunk + chunk) * k + threadIdx.x] = h[threadIdx.x];
}

// One CTA per head: base(chunk, c) = sum of all tokens of clusters < c plus the
// tokens of cluster c in earlier chunks.
__global__ void sort_scan_kernel(const int* __restrict__ ccount, int* __restrict__ cbase,
                                 int* __restrict__ counts, int* __restrict__ cstart, int k, int nchunk) {
  __shared__ int tot[VCA_MAX_CLUSTERS];
  __shared__ int off[VCA_MAX_CLUSTERS];
  const int bh = blockIdx.x, c = threadIdx.x;
  const int* cc = ccount + (int64_t)bh * nchunk * k;
  int* cb = cbase + (int64_t)bh * nchunk * k;
  if (c < k) {
    int s = 0;
    for (int j = 0; j < nchunk; ++j) s += cc[j * k + c];
    tot[c] = s;
  }
  __syncthreads();
  if (c == 0) {
    int run = 0;
    for (int i = 0; i < k; ++i) {
      off[i] = run;
      run += tot[i];
    }
  }
  __syncthreads();
  if (c < k) {
    counts[(int64_t)bh * k + c] = tot[c];
    cstart[(int64_t)bh * k + c] = off[c];
    int run = off[c];
    for (int j = 0; j < nchunk; ++j) {
      cb[j * k + c] = run;
      run += cc[j * k + c];
    }
  }
}

// One warp per chunk: tokens in index order, ranked inside each group of 32
// by matching cluster ids, so equal clusters keep their original order.
__global__ void __launch_bounds__(32) sort_scatter_kernel(const int32_t* __restrict__ assign,
                                                         const int* __restrict__ cbase,
                                                         int32_t* __restrict__ perm, int N, int k,
                                                         int nchunk) {
  __shared__ int base[VCA_MAX_CLUSTERS];
  const int bh = blockIdx.y, chunk = blockIdx.x, lane = threadIdx.x;
  for (int c = lane; c < k; c += 32) base[c] = cbase[((int64_t)bh * nchunk + chunk) * k + c];
  __syncwarp();
  const int n0 = chunk * kSortChunk, n1 = min(N, n0 + kSortChunk);
  const int32_t* ab = assign + (int64_t)bh * N;
  int32_t* pb = perm + (int64_t)bh * N;
  const unsigned lt = (1u << lane) - 1u;
  for (int g = n0; g < n1; g += 32) {
    int n = g + lane;
    bool valid = n < n1;
    unsigned active = __ballot_sync(0xffffffffu, valid);
    int a = valid ? ab[n] : -1 - lane;     // invalid lanes never match a cluster
    unsigned peers = __match_any_sync(0xffffffffu, a);
    int pos = 0;
    if (valid) pos = base[a] + __popc(peers & lt);
    __syncwarp();
    if (valid) {
      pb[pos] = n;
      if ((peers & lt) == 0) base[a] += __popc(peers & active);
    }
    __syncwarp();
  }
}

}  // namespace vca

using namespace vca;

extern "C" size_t vca_cluster_permute_workspace_size(int B, int H, int N, int k) {
  if (B < 1 || H < 1 || N < 1 || k < 1) return 0;
  size_t total;
  carve(nullptr, B * H, N, k, &total);
  return total;
}

static int cluster_permute_impl(const vca_bf16* V, int B, int H, int N, int d, int k, int iters,
                                const float* init, float* cent, int32_t* assign, int32_t* perm,
                                const KmWs& w, cudaStream_t s) {
  const int BH = B * H;
  size_t sums_bytes = (size_t)BH * k * 128 * sizeof(long long);
  km_init_kernel<<<dim3(BH, k), 128, 0, s>>>(V, init, cent, N, k);
  int rc = check_launch("km_init_kernel");
  if (rc) return rc;
  // the assignment's V tiles by TMA: [BH][N][128] bf16, 64 channels x 128 tokens
  // per box, so tokens past N read as zero and are not written
  AsgParams ap;
  {
    const uint64_t dims[3] = {128, (uint64_t)N, (uint64_t)BH}, str[2] = {256, (uint64_t)N * 256};
    const uint32_t box[3] = {64, 128, 1};
    rc = encode_tiled(&ap.tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  ap.cent = cent;
  ap.assign = assign;
  ap.st = w.st;
  ap.lim = wait_limit_ns();
  ap.N = N;
  ap.k = k;
  const int kp = k <= 32 ? 32 : 64;
  const size_t assign_smem = 1024 + 32768 + (size_t)4 * kp * 128;
  auto assign_kernel = kp == 32 ? km_assign_kernel<32> : km_assign_kernel<64>;
  if (cudaFuncSetAttribute(assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)assign_smem) !=
      cudaSuccess)
    return fail(VCA_ERR_CUDA, "vca_cluster_permute: cannot set shared-memory size");
  // persistent over a head's tiles: about 3 CTAs per SM over the whole layer, so
  // one wave (and at least one CTA per head)
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = (N + 127) / 128;
  int per_head = 3 * sms / BH;
  per_head = per_head < 1 ? 1 : (per_head > ntiles ? ntiles : per_head);
  const dim3 g_assign(per_head, BH);
  const dim3 g_accum((N + kSegWarps * kSegTok - 1) / (kSegWarps * kSegTok), BH);
  const int nchunk = (N + kSortChunk - 1) / kSortChunk;
  // Every round: assign, stable counting sort by cluster (its scan also gives
  // the cluster sizes and starts), exact sums along the sorted order, update.
  // The last round's sort is the permutation the caller gets.
  for (int it = 0; it < iters; ++it) {
    assign_kernel<<<g_assign, kAsgThreads, assign_smem, s>>>(ap);
    if ((rc = check_launch("km_assign_kernel"))) return rc;
    sort_count_kernel<<<dim3(nchunk, BH), 256, 0, s>>>(assign, w.ccount, N, k, nchunk);
    if ((rc = check_launch("sort_count_kernel"))) return rc;
    sort_scan_kernel<<<BH, 64, 0, s>>>(w.ccount, w.cbase, w.counts, w.cstart, k, nchunk);
    if ((rc = check_launch("sort_scan_kernel"))) return rc;
    sort_scatter_kernel<<<dim3(nchunk, BH), 32, 0, s>>>(assign, w.cbase, perm, N, k, nchunk);
    if ((rc = check_launch("sort_scatter_kernel"))) return rc;
    if (cudaMemsetAsync(w.sums, 0, sums_bytes, s) != cudaSuccess)
      return fail(VCA_ERR_CUDA, "vca_cluster_permute: memset failed");
    km_accum_kernel<<<g_accum, kSegWarps * 32, 0, s>>>(V, perm, w.cstart, w.counts, w.sums, N, k, w.st);
    if ((rc = check_launch("km_accum_kernel"))) return rc;
    km_update_kernel<<<dim3(BH, k), 128, 0, s>>>(w.sums, w.counts, cent, k);
    if ((rc = check_launch("km_update_kernel"))) return rc;
  }
  return 0;
}

static int check_cluster_args(const vca_bf16* V, int B, int H, int N, int d, int k, int iters,
                              const float* init, float* cent, int32_t* assign, int32_t* perm) {
  if (d != VCA_HEAD_DIM) return fail(VCA_ERR_UNSUPPORTED, "vca_cluster_permute: d must be 128");
  if (k < 1 || k > VCA_MAX_CLUSTERS)
    return fail(VCA_ERR_UNSUPPORTED, "vca_cluster_permute: k must be in [1, %d]", VCA_MAX_CLUSTERS);
  if (iters < 1 || iters > 64) return fail(VCA_ERR_INVALID, "vca_cluster_permute: iters must be in [1, 64]");
  if (B < 1 || H < 1 || N < 1 || (int64_t)B * H > 65535 || N > (1 << 24))
    return fail(VCA_ERR_INVALID, "vca_cluster_permute: bad shape B=%d H=%d N=%d", B, H, N);
  if (!V || !cent || !assign || !perm) return fail(VCA_ERR_INVALID, "vca_cluster_permute: null pointer");
  if (!aligned16(V) || !aligned16(cent) || (init && !aligned16(init)) || !aligned16(assign) || !aligned16(perm))
    return fail(VCA_ERR_INVALID, "vca_cluster_permute: pointers must be 16-byte aligned");
  return VCA_OK;
}

extern "C" int vca_cluster_permute(const vca_bf16* V, int B, int H, int N, int d, int k, int iters,
                                   const float* init_centroids, float* centroids, int32_t* assign,
                                   int32_t* perm, void* ws, size_t ws_bytes, vca_stream_t stream) {
  int rc = check_cluster_args(V, B, H, N, d, k, iters, init_centroids, centroids, assign, perm);
  if (rc) return rc;
  size_t need = vca_cluster_permute_workspace_size(B, H, N, k);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(VCA_ERR_WORKSPACE, "vca_cluster_permute: workspace needs %zu bytes", need);
  size_t total;
  KmWs w = carve(ws, B * H, N, k, &total);
  return cluster_permute_impl(V, B, H, N, d, k, iters, init_centroids, centroids, assign, perm, w,
                              (cudaStream_t)stream);
}

// ---------------------------------------------------------------- no-allocation variant
//
// Some callers cannot allocate device memory at the moment they run the
// grouping step: a plugin invoked from an engine that owns and budgets all GPU
// memory itself, or a latency-critical enqueue path where cudaMalloc may
// synchronise the device and stall other streams.  For them the scratch lives in
// one fixed array below, reserved on every GPU that loads this library until the
// process exits.  All calls share it, so calls whose kernels overlap on the GPU
// (other streams, other threads) race; serialise them on one stream.

static __device__ __align__(256) unsigned char g_cluster_scratch[VCA_NOALLOC_SCRATCH_BYTES];

// The array's device address, looked up on every call (the lookup allocates
// nothing, and after a device reset the address may differ) with the
// caller's device current.
static int noalloc_scratch(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_cluster_scratch);
  if (e != cudaSuccess || !p)
    return fail(VCA_ERR_CUDA, "vca_cluster_permute_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
  *out = p;
  return VCA_OK;
}

extern "C" int vca_cluster_permute_noalloc(const vca_bf16* V, int B, int H, int N, int d, int k, int iters,
                                           const float* init_centroids, float* centroids, int32_t* assign,
                                           int32_t* perm, vca_stream_t stream) {
  int rc = check_cluster_args(V, B, H, N, d, k, iters, init_centroids, centroids, assign, perm);
  if (rc) return rc;
  size_t need = vca_cluster_permute_workspace_size(B, H, N, k);
  if (need > (size_t)VCA_NOALLOC_SCRATCH_BYTES)
    return fail(VCA_ERR_UNSUPPORTED,
                "vca_cluster_permute_noalloc: B=%d H=%d N=%d k=%d needs %zu bytes of scratch, more than the "
                "fixed %zu; use vca_cluster_permute with a workspace",
                B, H, N, k, need, (size_t)VCA_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  // the array keeps the previous call's contents: its status word (where the
  // k-means kernels record out-of-range input) is cleared here; the sums and
  // counts are cleared before every k-means round and the sort tables are
  // written in full before they are read
  if (cudaMemsetAsync(scratch, 0, sizeof(DevStatus), (cudaStream_t)stream) != cudaSuccess)
    return fail(VCA_ERR_CUDA, "vca_cluster_permute_noalloc: cudaMemsetAsync failed");
  size_t total;
  KmWs w = carve(scratch, B * H, N, k, &total);
  return cluster_permute_impl(V, B, H, N, d, k, iters, init_centroids, centroids, assign, perm, w,
                              (cudaStream_t)stream);
}
