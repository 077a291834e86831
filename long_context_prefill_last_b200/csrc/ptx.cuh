// Device helpers: bounded mbarrier waits, TMA, tcgen05 (UMMA / TMEM), bf16.
// Inline PTX for sm_100a. No cluster multicast form of any copy is used.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace crisp {
namespace dev {

// ------------------------------------------------------------------ status word

// Record the first device-side error in the workspace status word.
__device__ __forceinline__ void report(int32_t* status, int code, int info) {
  if (status == nullptr) return;
  if (atomicCAS(status, 0, code) == 0) {
    status[1] = info;
  }
}

__device__ __forceinline__ int load_volatile(const int32_t* p) {
  return *reinterpret_cast<const volatile int32_t*>(p);
}

// ------------------------------------------------------------------ smem / mbarrier

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Cycles after which a wait is declared hung (about 0.5-1 s at B200 clocks).
constexpr long long kWaitLimitCycles = 1000000000LL;

// Bounded wait on phase `parity` of an mbarrier. Returns false (and raises
// the CTA abort flag and the global status) if the wait ran out, or if the
// abort flag or the global status was already set.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* gstatus, int where, long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0u) {
      if (*abort_flag) return false;
      if (load_volatile(gstatus) != 0) {
        *abort_flag = 1;
        return false;
      }
      if (clock64() - t0 > limit) {
        *abort_flag = 1;
        report(gstatus, CRISP_ERR_TIMEOUT, where);
        return false;
      }
    }
  }
}

// Bounded wait that ignores the abort flag (used to drain copies in flight
// before a CTA exits on the error path).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// 3-D tiled bulk tensor load global -> shared, completion on an mbarrier.
// x (innermost coordinate) must be a multiple of 8 bf16 / 4 fp32 elements.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(dst), "l"(tmap), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ------------------------------------------------------------------ tcgen05 / TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
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

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once every tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Warp-wide forms: the whole warp executes them (so the descriptors stay
// warp-uniform) and one elected lane issues the instruction.
//
// Eight K = 16 steps of D (+)= A * B with A and B K-major, 128-byte swizzled
// in shared memory (a 128 x 128 bf16 operand as two 64-column halves): step kk
// starts (kk / 4) halves and (kk % 4) * 32 bytes in, i.e. the descriptors'
// start-address fields (16-byte units) advance by (kk / 4) * 1024 + (kk % 4) * 2.
// The first step accumulates when `accumulate` is nonzero, the rest always.
#define CRISP_SS_STEP(OFF) \
  "add.s64 a, %1, " #OFF ";\n\tadd.s64 b, %2, " #OFF ";\n\t@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, pt;\n\t"
__device__ __forceinline__ void umma_ss8_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p0, pt;\n\t.reg .b32 r;\n\t.reg .b64 a, b;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 p0, %4, 0;\n\t"
      "setp.eq.b32 pt, %4, %4;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p0;\n\t"
      CRISP_SS_STEP(2) CRISP_SS_STEP(4) CRISP_SS_STEP(6) CRISP_SS_STEP(1024)
      CRISP_SS_STEP(1026) CRISP_SS_STEP(1028) CRISP_SS_STEP(1030)
      "}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
#undef CRISP_SS_STEP

// Eight K = 16 steps of D (+)= A * B with A in tensor memory (bf16 pairs, 8
// columns per step) and B MN-major, 128-byte swizzled in shared memory (16
// K-rows of 128 bytes per step: the start-address field advances by 128).
#define CRISP_TS_STEP(COL, OFF) \
  "add.u32 t, %1, " #COL ";\n\tadd.s64 b, %2, " #OFF ";\n\t@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, pt;\n\t"
__device__ __forceinline__ void umma_ts8_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p0, pt;\n\t.reg .b32 r, t;\n\t.reg .b64 b;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 p0, %4, 0;\n\t"
      "setp.eq.b32 pt, %4, %4;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
      CRISP_TS_STEP(8, 128) CRISP_TS_STEP(16, 256) CRISP_TS_STEP(24, 384) CRISP_TS_STEP(32, 512)
      CRISP_TS_STEP(40, 640) CRISP_TS_STEP(48, 768) CRISP_TS_STEP(56, 896)
      "}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
#undef CRISP_TS_STEP

// Eight K = 16 steps of D (+)= A * B with A in tensor memory (bf16 pairs, 8
// columns per step) and B K-major, 128-byte swizzled in shared memory (as in
// umma_ss8_w: (kk / 4) * 1024 + (kk % 4) * 2 in the start-address field).
#define CRISP_TSK_STEP(COL, OFF) \
  "add.u32 t, %1, " #COL ";\n\tadd.s64 b, %2, " #OFF ";\n\t@e tcgen05.mma.cta_group::1.kind::f16 [%0], [t], b, %3, pt;\n\t"
__device__ __forceinline__ void umma_ts8k_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p0, pt;\n\t.reg .b32 r, t;\n\t.reg .b64 b;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 p0, %4, 0;\n\t"
      "setp.eq.b32 pt, %4, %4;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n\t"
      CRISP_TSK_STEP(8, 2) CRISP_TSK_STEP(16, 4) CRISP_TSK_STEP(24, 6) CRISP_TSK_STEP(32, 1024)
      CRISP_TSK_STEP(40, 1026) CRISP_TSK_STEP(48, 1028) CRISP_TSK_STEP(56, 1030)
      "}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
#undef CRISP_TSK_STEP

// Commit (warp-wide form): one elected lane arrives on the mbarrier once every
// tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void umma_commit_w(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

// Instruction descriptor: bf16 x bf16 -> fp32, M x N, A K-major, B K-major or MN-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4)                          // D format: f32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16)   // B major
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle (the layout TMA writes
// with CU_TENSOR_MAP_SWIZZLE_128B: rows of 128 bytes, 16-byte chunks XORed
// with row % 8, 8-row groups of 1024 bytes).
//   K-major operand:  sbo = 1024 (next 8 rows), lbo unused (1)
//   MN-major operand: sbo = 1024 (next 8 K-rows), lbo = byte distance to the next 64 MN elements
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;   // layout: SWIZZLE_128B
  return d;
}

// 32 lanes x 32 columns of 32-bit TMEM -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Four 32-column loads issued back to back (one wait for all of them).
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float (&x)[128]) {
  uint32_t (&r)[128] = reinterpret_cast<uint32_t (&)[128]>(x);
  tmem_ld32(taddr, reinterpret_cast<uint32_t (&)[32]>(r[0]));
  tmem_ld32(taddr + 32, reinterpret_cast<uint32_t (&)[32]>(r[32]));
  tmem_ld32(taddr + 64, reinterpret_cast<uint32_t (&)[32]>(r[64]));
  tmem_ld32(taddr + 96, reinterpret_cast<uint32_t (&)[32]>(r[96]));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ math

// Hardware base-2 exponential (MUFU), flushes denormals; exp2(-inf) = 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA and integer pipes (no MUFU). x = n + f with n = round(x):
// adding 1.5 * 2^23 leaves round(x) in the low mantissa bits (Cody-Waite
// style reduction), f = x - n lies in [-1/2, 1/2]; 2^f is a minimax
// polynomial fitted by csrc/fit_exp2.py (Remez, relative error); 2^n is added
// to the exponent field. x is clamped to >= -125 so the result stays normal.
// Degree 3: relative error 7.5e-5 (ample for bf16 probabilities).
__device__ __forceinline__ float exp2_poly3(float x) {
  x = fmaxf(x, -125.f);
  const float shifter = 12582912.f;
  const float y = x + shifter;
  const float f = x - (y - shifter);
  float p = fmaf(0.0551716685f, f, 0.242611125f);
  p = fmaf(p, f, 0.693260968f);
  p = fmaf(p, f, 0.999928057f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(y) << 23));
}

// Degree 5: relative error 2.3e-7 in float32 (for sums that feed thresholds).
__device__ __forceinline__ float exp2_poly5(float x) {
  x = fmaxf(x, -125.f);
  const float shifter = 12582912.f;
  const float y = x + shifter;
  const float f = x - (y - shifter);
  float p = fmaf(0.00132764725f, f, 0.00967554096f);
  p = fmaf(p, f, 0.0555071309f);
  p = fmaf(p, f, 0.240221202f);
  p = fmaf(p, f, 0.693146944f);
  p = fmaf(p, f, 1.00000012f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(y) << 23));
}

// ---- packed pairs of fp32 (Blackwell f32x2 arithmetic: one instruction, two lanes of work)
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// exp2_poly3 on a packed pair (same reduction and polynomial as exp2_poly3);
// the caller clamps both inputs to >= -125.
__device__ __forceinline__ void exp2_poly3_x2(uint64_t x2, float& p0, float& p1) {
  const uint64_t shift = f2_pack(12582912.f, 12582912.f);
  const uint64_t nshift = f2_pack(-12582912.f, -12582912.f);
  const uint64_t minus1 = f2_pack(-1.f, -1.f);
  const uint64_t y = f2_add(x2, shift);
  const uint64_t f = f2_fma(f2_add(y, nshift), minus1, x2);   // x - round(x)
  uint64_t p = f2_fma(f2_pack(0.0551716685f, 0.0551716685f), f, f2_pack(0.242611125f, 0.242611125f));
  p = f2_fma(p, f, f2_pack(0.693260968f, 0.693260968f));
  p = f2_fma(p, f, f2_pack(0.999928057f, 0.999928057f));
  float y0, y1;
  f2_unpack(y, y0, y1);
  f2_unpack(p, p0, p1);
  p0 = __int_as_float(__float_as_int(p0) + (__float_as_int(y0) << 23));
  p1 = __int_as_float(__float_as_int(p1) + (__float_as_int(y1) << 23));
}

// Register split between warpgroups (all four warps of a warpgroup execute it).
template <int N>
__device__ __forceinline__ void regs_release() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_acquire() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ bool mask_bit(const uint32_t* m, int b) { return (m[b >> 5] >> (b & 31)) & 1u; }

// Tile classes of the attention schedule.
enum TileKind : int { kSkip = 0, kFull = 1, kLower = 2 /* keep c <= r */, kUpper = 3 /* keep c > r */ };

// Which part of key tile t a query tile I needs (t <= I).
//   VS: key j kept when its column block is selected, or its offset block
//       (i - j) / B is: inside tile (I, t) the offsets of c <= r lie in block
//       I - t and those of c > r in block I - t - 1.
//   PE: the whole tile when block (I, t) is selected; the diagonal always.
//   dense: every tile; the diagonal tile is causal.
__device__ __forceinline__ int tile_kind(int route, const uint32_t* vmask, const uint32_t* smask,
                                         const uint32_t* pe_row, bool dense, int I, int t) {
  if (t == I) return kLower;
  if (dense) return kFull;
  if (route == 1) return mask_bit(pe_row, t) ? kFull : kSkip;
  if (mask_bit(vmask, t)) return kFull;
  const bool lo = mask_bit(smask, I - t);
  const bool hi = mask_bit(smask, I - t - 1);
  if (lo && hi) return kFull;
  if (lo) return kLower;
  if (hi) return kUpper;
  return kSkip;
}

}  // namespace dev
}  // namespace crisp
