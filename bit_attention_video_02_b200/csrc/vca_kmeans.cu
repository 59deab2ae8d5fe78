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
// per channel, so the argmin is reproducible bit for bit), accumulate
// (channel-parallel exact 2^-24 fixed-point sums in int64, order-free), update
// (one fp64 division per centroid coordinate).  Then a stable counting sort:
// per-chunk histograms, an exclusive scan in (cluster, chunk) order, and a
// warp-synchronous ranked scatter.
#include <mutex>

#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

constexpr int kAssignThreads = 128;
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

// Shared-memory centroid table for the assignment: pairs of centroids
// interleaved per channel and negated, cs[p][ch] = (-mu_{2p}[ch], -mu_{2p+1}[ch]),
// so one fma.rn.f32x2 advances the distances to two centroids.  An odd k is
// padded with a centroid at infinity, which never wins.  The channel loop is
// outside the centroid loop, so each bf16 channel is unpacked once per token
// and feeds NP accumulator pairs; every accumulator still adds its channels
// in order 0..127 (the distance's defined summation order).
template <int NP>
__global__ void __launch_bounds__(kAssignThreads) km_assign_kernel(const uint16_t* __restrict__ V,
                                                                  const float* __restrict__ cent,
                                                                  int32_t* __restrict__ assign,
                                                                  int N, int k) {
  extern __shared__ float4 cs4[];   // [NP][64] float4 = [pairs][128 channels][2]
  const int bh = blockIdx.y;
  const int npairs = (k + 1) >> 1;
  const float* src = cent + (int64_t)bh * k * 128;
  float2* cs2 = reinterpret_cast<float2*>(cs4);
  for (int i = threadIdx.x; i < NP * 128; i += blockDim.x) {
    const int pp = i >> 7, ch = i & 127, c0 = 2 * pp, c1 = 2 * pp + 1;
    cs2[i] = make_float2(c0 < k ? -src[c0 * 128 + ch] : -INFINITY, c1 < k ? -src[c1 * 128 + ch] : -INFINITY);
  }
  __syncthreads();
  // two tokens per thread (n and n + blockDim.x): every centroid value read from
  // shared memory serves both
  const int n = blockIdx.x * 2 * blockDim.x + threadIdx.x, nb2 = n + blockDim.x;
  if (n >= N) return;
  const bool has_b = nb2 < N;
  const uint4* row = reinterpret_cast<const uint4*>(V + ((int64_t)bh * N + n) * 128);
  const uint4* rowb = reinterpret_cast<const uint4*>(V + ((int64_t)bh * N + (has_b ? nb2 : n)) * 128);
  float2 acc[NP], accb[NP];
#pragma unroll
  for (int pp = 0; pp < NP; ++pp) acc[pp] = accb[pp] = make_float2(0.0f, 0.0f);
  // 8 channels per step; the next 16-byte pieces of the rows are loaded one step ahead
  uint4 cur = __ldg(row), curb = __ldg(rowb);
#pragma unroll 1
  for (int q = 0; q < 16; ++q) {
    const int qn = q + 1 < 16 ? q + 1 : q;
    const uint4 nxt = __ldg(row + qn), nxtb = __ldg(rowb + qn);
    const uint32_t w[4] = {cur.x, cur.y, cur.z, cur.w}, wb[4] = {curb.x, curb.y, curb.z, curb.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = 4 * q + u;   // channels 2i, 2i+1
      const float x0 = __uint_as_float(w[u] << 16), x1 = __uint_as_float(w[u] & 0xFFFF0000u);
      const float y0 = __uint_as_float(wb[u] << 16), y1 = __uint_as_float(wb[u] & 0xFFFF0000u);
      const float2 X0 = make_float2(x0, x0), X1 = make_float2(x1, x1);
      const float2 Y0 = make_float2(y0, y0), Y1 = make_float2(y1, y1);
#pragma unroll
      for (int pp = 0; pp < NP; ++pp) {
        const float4 m = cs4[pp * 64 + i];   // channels 2i (x, y) and 2i+1 (z, w)
        const float2 m0 = make_float2(m.x, m.y), m1 = make_float2(m.z, m.w);
        float2 t = __fadd2_rn(X0, m0);   // v - mu, exact order per lane
        acc[pp] = __ffma2_rn(t, t, acc[pp]);
        t = __fadd2_rn(X1, m1);
        acc[pp] = __ffma2_rn(t, t, acc[pp]);
        t = __fadd2_rn(Y0, m0);
        accb[pp] = __ffma2_rn(t, t, accb[pp]);
        t = __fadd2_rn(Y1, m1);
        accb[pp] = __ffma2_rn(t, t, accb[pp]);
      }
    }
    cur = nxt;
    curb = nxtb;
  }
  int best = 0, bestb = 0;
  float bd = acc[0].x, bdb = accb[0].x;
#pragma unroll
  for (int pp = 0; pp < NP; ++pp) {
    if (pp > 0 && acc[pp].x < bd) {
      bd = acc[pp].x;
      best = 2 * pp;
    }
    if (acc[pp].y < bd) {
      bd = acc[pp].y;
      best = 2 * pp + 1;
    }
    if (pp > 0 && accb[pp].x < bdb) {
      bdb = accb[pp].x;
      bestb = 2 * pp;
    }
    if (accb[pp].y < bdb) {
      bdb = accb[pp].y;
      bestb = 2 * pp + 1;
    }
  }
  if (has_b) assign[(int64_t)bh * N + nb2] = bestb;
  (void)npairs;
  assign[(int64_t)bh * N + n] = best;
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
  // centroid table padded to 16 or 32 pairs (pads sit at infinity)
  const int np = (k + 1) / 2 <= 16 ? 16 : 32;
  const size_t assign_smem = (size_t)np * 128 * sizeof(float2);
  auto assign_kernel = np == 16 ? km_assign_kernel<16> : km_assign_kernel<32>;
  if (cudaFuncSetAttribute(assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)assign_smem) !=
      cudaSuccess)
    return fail(VCA_ERR_CUDA, "vca_cluster_permute: cannot set shared-memory size");
  const dim3 g_assign((N + 2 * kAssignThreads - 1) / (2 * kAssignThreads), BH);
  const dim3 g_accum((N + kSegWarps * kSegTok - 1) / (kSegWarps * kSegTok), BH);
  const int nchunk = (N + kSortChunk - 1) / kSortChunk;
  // Every round: assign, stable counting sort by cluster (its scan also gives
  // the cluster sizes and starts), exact sums along the sorted order, update.
  // The last round's sort is the permutation the caller gets.
  for (int it = 0; it < iters; ++it) {
    assign_kernel<<<g_assign, kAssignThreads, assign_smem, s>>>(V, cent, assign, N, k);
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
