// sm100_ptx.cuh -- thin inline-PTX wrappers for the sm_100a features the attention
// kernels use: mbarriers (with bounded waits), TMA tensor copies, and the fifth-
// generation tensor cores (tcgen05 MMA with accumulators in tensor memory).
//
// Every wait here is bounded: a pipeline wait that exceeds kWaitLimitCycles (about two
// seconds) or sees the CTA's abort flag returns false instead of spinning on, so a
// broken pipeline ends with an error status rather than a hung GPU.  The waits with
// which a failing CTA collects its own copies and MMAs before it exits have their own,
// fixed limit (kDrainLimitCycles).  A test build of the library shortens the pipeline
// limit (FA_WAIT_LIMIT_CYCLES) so that every pipeline runs out and takes its error path.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#ifndef FA_WAIT_LIMIT_CYCLES
#define FA_WAIT_LIMIT_CYCLES 4000000000LL
#endif

namespace fa {

constexpr long long kWaitLimitCycles = FA_WAIT_LIMIT_CYCLES;
constexpr long long kDrainLimitCycles = 4000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// The suspend-time hint (20 us) lets a waiting warp sleep until the phase completes
// instead of polling and taking issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
// Waits for the phase of `bar` with the given parity to complete.  Returns false
// (without completing) when the CTA's abort flag is raised or the time limit passes.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
}
// Non-blocking test of a phase.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Like mbar_wait, but polls without ever suspending the warp: for the single MMA-issuing
// thread, which should react to a completed phase at once (the many softmax warps use
// mbar_wait, whose suspension keeps their polling off the shared-memory pipe).
__device__ __forceinline__ bool mbar_wait_spin(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_test_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_test_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
}
// Same, ignoring the abort flag and with the fixed drain limit (used to collect a CTA's own
// in-flight copies and MMAs on the way out).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > kDrainLimitCycles) return false;
  }
}

// ----------------------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tm) : "memory");
}
// 3-D tiled load global -> shared, completion signalled as transaction bytes on `bar`.
// The innermost coordinate x is always a multiple of 64 elements (128 bytes) here.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(tm), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// 3-D tiled store shared -> global (rows outside the tensor are clipped by the hardware).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* tm, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(tm),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Makes this thread's generic-proxy shared-memory writes visible to the async proxy (TMA, MMA).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Untiled bulk copy global -> shared (both addresses and the size multiples of 16 bytes).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// ----------------------------------------------------------------------------- tensor memory
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive (once) on `bar` when every tcgen05 op this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 x bf16 -> fp32.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T, A read from tensor memory (one row per lane).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Four K-steps of one product, issued back to back from precomputed descriptors: step k
// (k = 0..3) uses the A and B descriptors advanced by the k-th offsets (step 0: none), in
// the descriptors' 16-byte start-address units.  The sums stay inside the 14-bit
// start-address field since every shared-memory address here is below 256 KB.  Only
// step 0 honours `accumulate`; steps 1..3 always accumulate.  The MMA-issuing thread
// shares its SMSP with busy element-wise warps, so every instruction it saves per MMA
// shortens the gaps in which the tensor pipe waits for work.
template <int A1, int A2, int A3, int B1, int B2, int B3>
__device__ __forceinline__ void mma_ss_x4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "add.s64 a, %1, %6;\n\tadd.s64 b, %2, %9;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n\t"
      "add.s64 a, %1, %7;\n\tadd.s64 b, %2, %10;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n\t"
      "add.s64 a, %1, %8;\n\tadd.s64 b, %2, %11;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(1u), "n"(A1), "n"(A2), "n"(A3), "n"(B1), "n"(B2),
      "n"(B3)
      : "memory");
}
// Same with A read from tensor memory: the A offsets are tensor-memory columns.
template <int A1, int A2, int A3, int B1, int B2, int B3>
__device__ __forceinline__ void mma_ts_x4(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b32 a;\n\t.reg .b64 b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "add.s32 a, %1, %6;\n\tadd.s64 b, %2, %9;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n\t"
      "add.s32 a, %1, %7;\n\tadd.s64 b, %2, %10;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n\t"
      "add.s32 a, %1, %8;\n\tadd.s64 b, %2, %11;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(1u), "n"(A1), "n"(A2), "n"(A3), "n"(B1), "n"(B2),
      "n"(B3)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets row (lane base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// After tmem_ld_wait(): ties the loaded registers to a point after the wait, so the
// compiler cannot schedule their uses before the data has arrived.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// ----------------------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 "version 1" format):
// start address, leading- and stride-dimension byte offsets (all >> 4).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version for sm_100
  d |= (uint64_t)2 << 61;   // layout: 128-byte swizzle
  return d;
}
// Instruction descriptor, kind::f16 with bf16 (or, when f16, fp16) A and B and fp32
// accumulate, dense.  a_mn / b_mn select MN-major (transposed) operands.
__host__ __device__ constexpr uint32_t idesc_16(int M, int N, bool a_mn, bool b_mn, bool f16) {
  return (1u << 4)                      // D format: f32
         | ((f16 ? 0u : 1u) << 7)       // A format: f16 (0) or bf16 (1)
         | ((f16 ? 0u : 1u) << 10)      // B format: same type as A
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ----------------------------------------------------------------------------- math
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Maximum that propagates NaN (max.NaN.f32): max(NaN, y) is NaN, max(-inf, y) is y.
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
// 2^x for two values at once on the FMA pipe (packed fp32x2 arithmetic), so that part
// of the exponentials can bypass the MUFU unit.  Cody-Waite range reduction
// (x = n + f, n = round(x) by adding 1.5*2^23 + 127 so that the sum's low mantissa
// bits hold n + 127, f in [-1/2, 1/2]), a cubic for 2^f whose coefficients minimise
// the maximum relative error on [-1/2, 1/2] (Remez exchange; derived by
// gen_exp2_poly.py in this directory), and 2^n, built from those low bits as a
// float's exponent field, applied by one multiplication.  Max relative error 7.8e-5
// for x in [-125, 10]; x below -125 (including -inf) is clamped to -125, i.e. a
// result of ~2.4e-38.  NaN propagates as it does through MUFU ex2: the clamp keeps a
// NaN, the polynomial of a NaN is NaN, and NaN times the scale is NaN.
constexpr float kExp2C0 = 0.99992805719375610f;   // 0x3f7ffb49
constexpr float kExp2C1 = 0.69326096773147583f;   // 0x3f31798d
constexpr float kExp2C2 = 0.24261112511157990f;   // 0x3e786f0d
constexpr float kExp2C3 = 0.05517166852951050f;   // 0x3d61fbb0
constexpr float kExp2Round = 12583039.f;          // 1.5 * 2^23 + 127
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmax_nan(x.x, -125.f);
  x.y = fmax_nan(x.y, -125.f);
  const float2 t = __fadd2_rn(x, make_float2(kExp2Round, kExp2Round));
  const float2 n = __fadd2_rn(t, make_float2(-kExp2Round, -kExp2Round));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(f, make_float2(kExp2C3, kExp2C3), make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(kExp2C0, kExp2C0));
  const float2 scale = make_float2(__int_as_float(__float_as_int(t.x) << 23), __int_as_float(__float_as_int(t.y) << 23));
  return __fmul2_rn(p, scale);
}
// 2^x for a pair: on the FMA pipe when `poly`, else two MUFU ex2.approx.
__device__ __forceinline__ float2 exp2_pair(float2 x, bool poly) {
  return poly ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// Packs two floats to bf16x2 (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Same for fp16x2.
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// 16-bit element type of the kernels: bf16 or (F16) fp16, packed two per 32-bit word.
template <bool F16>
__device__ __forceinline__ uint32_t pack16(float lo, float hi) {
  return F16 ? pack_f16(lo, hi) : pack_bf16(lo, hi);
}
template <bool F16>
__device__ __forceinline__ float unpack16_lo(uint32_t x) {
  if (F16) return __half2float(__ushort_as_half(static_cast<unsigned short>(x & 0xffffu)));
  return __uint_as_float(x << 16);
}
template <bool F16>
__device__ __forceinline__ float unpack16_hi(uint32_t x) {
  if (F16) return __half2float(__ushort_as_half(static_cast<unsigned short>(x >> 16)));
  return __uint_as_float(x & 0xffff0000u);
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Four fp32 values added to global memory at `addr` (16-byte aligned) by the L2's
// reduction units; no value is returned, so the issuing thread does not wait.
__device__ __forceinline__ void red_add_f32x4(float* addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(__uint_as_float(a)),
               "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
               : "memory");
}

// Debug build (compiled with FA_DEBUG_CHECKS): device-side checks of every computed
// global-memory index and shared-memory offset against its buffer, and of warp convergence
// at the entry of each phase that issues warp-collective (.sync.aligned) tensor-memory
// operations.  A failed check records FA_ERR_DEBUG_CHECK in the status word and skips the
// guarded access, so a wrong index never touches memory outside its buffer.  In the normal
// build both macros compile to nothing.
constexpr int kStatusDebugCheck = 12;   // FA_ERR_DEBUG_CHECK
__device__ __forceinline__ bool debug_check(bool ok, int* status) {
  if (!ok && status != nullptr) atomicCAS(status, 0, kStatusDebugCheck);
  return ok;
}
#ifdef FA_DEBUG_CHECKS
#define FA_BOUNDS(cond, status) (::fa::debug_check(static_cast<bool>(cond), (status)))
#define FA_CONVERGED(status) ((void)::fa::debug_check(__activemask() == 0xffffffffu, (status)))
#else
#define FA_BOUNDS(cond, status) true
#define FA_CONVERGED(status) ((void)0)
#endif

// Records the first error code in the device status word and raises the CTA's abort flag.
__device__ __forceinline__ void raise_error(int* status, volatile int* abort_flag, int code) {
  *abort_flag = 1;
  atomicCAS(status, 0, code);
}

}  // namespace fa
