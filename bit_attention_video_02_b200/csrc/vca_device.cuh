// vca_device.cuh -- sm_100a device helpers for the vca kernels: error word,
// bounded mbarrier waits, TMA tile loads, tcgen05 (TMEM alloc, MMA, commit,
// TMEM load/store) and the shared-memory / instruction descriptors.
//
// Descriptor bit layouts follow the PTX ISA's tcgen05 "shared memory
// descriptor" and "instruction descriptor" tables (sm_100a).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vca.h"

namespace vca {

// ---------------------------------------------------------------- status word
// The first bytes of every caller workspace: the first device-side error wins.
struct DevStatus {
  int code;      // 0 = ok, else a VCA_ERR_* value
  int where;     // kernel-specific location tag
  int info;      // kernel-specific detail (block index, wait id, ...)
  int pad;
};

__device__ __forceinline__ void report(DevStatus* st, int code, int where, int info) {
  if (st && atomicCAS(&st->code, 0, code) == 0) {
    st->where = where;
    st->info = info;
  }
}

// ---------------------------------------------------------------- smem / sync
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete, for at most
// `limit_ns` nanoseconds of wall time.  On expiry it records VCA_ERR_TIMEOUT
// (with the wait's tag) and sets *abort so the other roles of the CTA stop;
// it also gives up at once when *abort is already set.  Returns true when the
// phase completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, DevStatus* st,
                                                  uint64_t limit_ns, int tag) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        report(st, VCA_ERR_TIMEOUT, tag, (int)blockIdx.x);
        *abort = 1;
        return false;
      }
    }
  }
}

// Warp-uniform form for code that follows with .sync.aligned tcgen05
// instructions: every lane waits, and the warp proceeds only if all lanes saw
// the phase complete (a lane that gave up makes the whole warp give up).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort,
                                               DevStatus* st, uint64_t limit_ns, int tag) {
  bool ok = mbar_wait_bounded(bar, parity, abort, st, limit_ns, tag);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}


// Warp-issued forms: the whole converged warp runs the issue loop in lockstep
// (so descriptors and addresses stay warp-uniform and cost one set of uniform
// instructions) and elect.sync picks the issuing lane -- lane 0 whenever all 32
// lanes are active, so MMAs and the commits that track them come from the same
// thread.
__device__ __forceinline__ void mma_tf32_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                              uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void mma_bf16_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                              uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void mma_bf16_ts_w(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                              uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void tc_commit_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

// The four 32-byte K steps of a K = 128 contraction of 8-bit operands and the
// commit that follows them, issued by one lane that a single elect.sync picks
// (one elect per group instead of one per instruction).  Step k reads the
// shared-memory descriptors advanced by 2k (16-byte units) and, for an A operand
// in tensor memory, the columns advanced by 8k; the first step accumulates iff
// accum0 != 0, the others always.  KIND is the tcgen05.mma kind as a string
// literal ("f8f6f4", "i8").
#define VCA_MMA4_SS_W(KIND, d, a, b, idesc, accum0, bar)                                            \
  asm volatile("{\n\t.reg .pred e, p0, p1;\n\t.reg .b64 a1, a2, a3, b1, b2, b3;\n\t"               \
               "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"                 \
               "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"                 \
               "setp.ne.b32 p0, %4, 0;\n\tsetp.eq.b32 p1, %4, %4;\n\t"                              \
               "elect.sync _|e, 0xffffffff;\n\t"                                                    \
               "@e tcgen05.mma.cta_group::1.kind::" KIND " [%0], %1, %2, %3, p0;\n\t"             \
               "@e tcgen05.mma.cta_group::1.kind::" KIND " [%0], a1, b1, %3, p1;\n\t"             \
               "@e tcgen05.mma.cta_group::1.kind::" KIND " [%0], a2, b2, %3, p1;\n\t"             \
               "@e tcgen05.mma.cta_group::1.kind::" KIND " [%0], a3, b3, %3, p1;\n\t"             \
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t}" \
               ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum0), "r"(smem_u32(bar))                \
               : "memory")
// The same for the block-scaled E4M3 x E4M3 MMA with A (the P codes) in tensor
// memory and the UE8M0 scale vectors at sfa / sfb.
#define VCA_MMA4_MXF8_TS_W(d, a_tmem, b, idesc, sfa, sfb, accum0, bar)                               \
  asm volatile("{\n\t.reg .pred e, p0, p1;\n\t.reg .b64 b1, b2, b3;\n\t.reg .b32 a1, a2, a3;\n\t"   \
               "add.s32 a1, %1, 8;\n\tadd.s32 a2, %1, 16;\n\tadd.s32 a3, %1, 24;\n\t"               \
               "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"                 \
               "setp.ne.b32 p0, %6, 0;\n\tsetp.eq.b32 p1, %6, %6;\n\t"                              \
               "elect.sync _|e, 0xffffffff;\n\t"                                                    \
               "@e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], [%1], %2, %3, [%4], [%5], p0;\n\t" \
               "@e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], [a1], b1, %3, [%4], [%5], p1;\n\t" \
               "@e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], [a2], b2, %3, [%4], [%5], p1;\n\t" \
               "@e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], [a3], b3, %3, [%4], [%5], p1;\n\t" \
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t}" \
               ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accum0),           \
                 "r"(smem_u32(bar))                                                                 \
               : "memory")

// 32 consecutive 32-bit TMEM columns of this thread's lane -> registers.
#define VCA_TMEM_LD32(taddr, r)                                                                  \
  asm volatile(                                                                                  \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"             \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),       \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),   \
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),            \
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),            \
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])             \
      : "r"(taddr))

#define VCA_TMEM_ST32(taddr, r)                                                                   \
  asm volatile(                                                                                   \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13," \
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(     \
          taddr),                                                                                 \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),     \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),          \
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),        \
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),        \
      "r"(r[29]), "r"(r[30]), "r"(r[31]))

#define VCA_TMEM_ST16(taddr, r)                                                               \
  asm volatile(                                                                               \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13," \
      "%14,%15,%16};" ::"r"(taddr),                                                           \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),      \
      "r"(r[15]))

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7]));
}
// One 32-bit TMEM column of this thread's lane (valid after tmem_ld_wait and
// reg_after_wait on the result).
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  return r;
}
// Pins a register loaded by an asynchronous tcgen05.ld after the wait that
// completes it, so no use of it is scheduled above that wait.
__device__ __forceinline__ void reg_after_wait(uint32_t& r) { asm volatile("" : "+r"(r)::"memory"); }
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (sm_100 format): start address >> 4 in bits
// [0,14), leading-dimension byte offset >> 4 in [16,30), stride-dimension byte
// offset >> 4 in [32,46), the fixed version value 1 in [46,48), base offset 0,
// layout type in [61,64) (0 none, 2 = 128-byte swizzle, 4 = 64B, 6 = 32B).
enum : uint32_t { kLayoutNone = 0, kLayoutSW128 = 2, kLayoutSW64 = 4, kLayoutSW32 = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// Instruction descriptor, dense kinds (f16 / tf32 / f8f6f4): D format in
// [4,6) (1 = f32), A format [7,10), B format [10,13), A major bit 15, B major
// bit 16 (1 = MN-major), N >> 3 in [17,23), M >> 4 in [24,29).
enum : uint32_t { kFmtE4M3 = 0, kFmtF16 = 0, kFmtBF16 = 1, kFmtTF32 = 2 };

__host__ __device__ constexpr uint32_t instr_desc(uint32_t afmt, uint32_t bfmt, int M, int N,
                                                  uint32_t a_mn_major, uint32_t b_mn_major) {
  return (1u << 4) | (afmt << 7) | (bfmt << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Integer kind (kind::i8): D format 2 (s32) in [4,6), A and B type 1 (signed
// 8-bit), no saturation (|sum| < 2^21 for 128 products of magnitude <= 127^2).
__host__ __device__ constexpr uint32_t instr_desc_s8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Block-scaled variant (kind::mxf8f6f4): B scale-factor id in [4,6), scale
// format bit 23 (1 = UE8M0), A scale-factor id in [29,31); no D-format field.
__host__ __device__ constexpr uint32_t instr_desc_mx(uint32_t afmt, uint32_t bfmt, int M, int N) {
  return (afmt << 7) | (bfmt << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- numerics

// bf16 halves of a 32-bit word as fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Round a double to bf16, nearest-even, in one step on the integer bits.
__device__ __forceinline__ uint16_t double_to_bf16_rne(double x) {
  unsigned long long b = (unsigned long long)__double_as_longlong(x);
  unsigned long long sign = b >> 63;
  unsigned long long a = b & 0x7FFFFFFFFFFFFFFFull;
  if (a == 0) return (uint16_t)(sign << 15);
  int e = (int)(a >> 52) - 1023;
  if (e >= -126) {
    // keep 7 fraction bits of the double's 52: round at bit 45
    unsigned long long lsb = (a >> 45) & 1ull;
    unsigned long long r = (a + 0x00000FFFFFFFFFFFull + lsb) >> 45;   // exponent | 7-bit fraction
    int e2 = (int)(r >> 7) - 1023;
    if (e2 > 127) return (uint16_t)((sign << 15) | 0x7F80u);
    return (uint16_t)((sign << 15) | ((unsigned)(e2 + 127) << 7) | (unsigned)(r & 0x7F));
  }
  // bf16 subnormal range: value = m * 2^-133, m in [0, 128]
  double m = rint(x < 0 ? -x * 0x1p133 : x * 0x1p133);
  return (uint16_t)((sign << 15) | (unsigned)m);
}

// Exact split of llrint(v * 2^24) for |v| < 2^20 (at most 45 bits) into
// hi * 2^22 + lo with |hi| < 2^22, |lo| <= 2^21, using float operations only:
// f = v * 2^24 is exact, hi = rne(f / 2^22) by the magic-number add (f / 2^22
// is exact), lo = rne(f - hi * 2^22) (the remainder is exact; its rounding is
// the only one, the same as llrint's since hi * 2^22 is an integer); each
// becomes an integer through the magic-number add.  No conversion instruction.
__device__ __forceinline__ void fix24_split(float v, int& hi, int& lo) {
  const float kMagic = 12582912.0f;   // 1.5 * 2^23
  const float f = v * 16777216.0f;
  const float hm = __fadd_rn(f * 2.384185791015625e-07f, kMagic);   // 1.5 * 2^23 + rne(f / 2^22)
  const float hf = __fsub_rn(hm, kMagic);
  const float lf = __fmaf_rn(hf, -4194304.0f, f);                   // exact remainder
  hi = (int)(__float_as_uint(hm) - 0x4B400000u);
  lo = (int)(__float_as_uint(lf + kMagic) - 0x4B400000u);
}

// Two fp32 -> two E4M3 bytes, round-to-nearest-even, saturating (hardware cvt).
// Result: low byte = e4m3(lo), next byte = e4m3(hi).
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}



// max of three fp32 values in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

}  // namespace vca
