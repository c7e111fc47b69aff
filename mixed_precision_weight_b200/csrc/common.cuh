// Device helpers shared by the DV-SSQ kernels (sm_100a).
//
// PTX wrappers for mbarriers, bulk/tensor copies, programmatic dependent
// launch, warp-level MMA and the 5th-generation tensor-core (tcgen05) ops,
// plus exact format conversions.  Every wait is bounded: after
// g_wait_limit cycles (kWaitLimitCycles unless the host shortened it) the
// waiter records an error code in g_dvssq_error and gives up, so that no
// kernel can hang the device.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dvssq {

// --------------------------------------------------------------- errors ---
enum DeviceError : uint32_t {
  kErrWaitMbarrier = 1u << 0,   // an mbarrier wait ran out
  kErrWaitTmem = 1u << 1,       // a TMEM accumulator wait ran out
  kErrBadShape = 1u << 2,       // a kernel saw a shape it does not support
  kErrWaitGrid = 1u << 3,       // a grid-wide barrier wait ran out
};

// Device error word of the library (one translation unit: see libdvssq.cu).
__device__ uint32_t g_dvssq_error = 0;

__device__ __forceinline__ void set_error(uint32_t code) { atomicOr(&g_dvssq_error, code); }

// ~2 s at 1.9 GHz: far beyond any legitimate wait, short enough to give up.
constexpr long long kWaitLimitCycles = 4000000000LL;

// The limit every bounded wait applies, in SM clock cycles.  The host sets
// it through dvssq_set_wait_limit (a test shortens it to make a wait run out).
__device__ long long g_wait_limit = kWaitLimitCycles;

__device__ __forceinline__ long long wait_limit() {
  return *(volatile long long *)&g_wait_limit;
}

// ------------------------------------------------------------ conversions -
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) {
  return __uint_as_float(b << 16);
}

// Round a double to the nearest BF16 (ties to even), returned as its bits.
// Written from the IEEE formats: keep 8 significand bits of the 53.
__device__ __forceinline__ uint16_t f64_to_bf16_rn(double x) {
  unsigned long long u = (unsigned long long)__double_as_longlong(x);
  uint32_t sign = (uint32_t)(u >> 63) << 15;
  unsigned long long a = u & 0x7FFFFFFFFFFFFFFFull;
  if (a >= 0x7FF0000000000000ull) {                 // inf or NaN
    return (uint16_t)(sign | (a == 0x7FF0000000000000ull ? 0x7F80u : 0x7FC0u));
  }
  int eb = (int)(a >> 52);
  if (eb == 0) return (uint16_t)sign;               // fp64 subnormal: far below bf16
  int e = eb - 1023;
  unsigned long long mant = (a & 0x000FFFFFFFFFFFFFull) | 0x0010000000000000ull;
  if (e >= -126) {
    unsigned long long keep = mant >> 45;           // 8 bits incl. hidden one
    unsigned long long rem = mant & ((1ull << 45) - 1);
    const unsigned long long half = 1ull << 44;
    if (rem > half || (rem == half && (keep & 1))) keep += 1;
    if (keep == 256) { keep = 128; e += 1; }
    if (e > 127) return (uint16_t)(sign | 0x7F80u);
    return (uint16_t)(sign | ((uint32_t)(e + 127) << 7) | (uint32_t)(keep & 0x7F));
  }
  // bf16 subnormal: quantum 2^-133; value = mant * 2^(e-52)
  int s = -81 - e;                                  // right shift to units of 2^-133
  if (s >= 64) return (uint16_t)sign;
  unsigned long long keep = mant >> s;
  unsigned long long rem = mant & ((1ull << s) - 1);
  unsigned long long half = 1ull << (s - 1);
  if (rem > half || (rem == half && (keep & 1))) keep += 1;
  return (uint16_t)(sign | (uint32_t)keep);         // keep == 128 -> smallest normal
}

__device__ __forceinline__ double bf16_bits_to_f64(uint32_t b) {
  return (double)__uint_as_float(b << 16);
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// --------------------------------------------------------- smem addresses -
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// gelu(v) = v/2 (1 + erf(v / sqrt 2)) in FP32.  1 + erf(z) = erfc(-z): the
// complementary form keeps its relative accuracy for negative v, where
// 1 + erf would cancel.
__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * erfcf(-v * 0.70710678118654752f);
}

// --------------------------------------------------------------- mbarrier -
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on phase `parity`; returns false (and flags the device error
// word) if the phase did not complete within the wait limit.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64(), lim = wait_limit();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > lim) {
      set_error(kErrWaitMbarrier);
      return false;
    }
  }
  return true;
}

// Bounded wait, by one thread, until the global counter reaches `target`
// (acquire).  Gives up, flags kErrWaitGrid and returns false when the wait
// limit runs out or when the device error word changes from `err0` (another
// CTA gave up first).
__device__ __forceinline__ bool counter_wait(const unsigned int *ctr, unsigned int target,
                                             uint32_t err0) {
  const long long t0 = clock64(), lim = wait_limit();
  while (true) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if (*(volatile uint32_t *)&g_dvssq_error != err0 || clock64() - t0 > lim) {
      set_error(kErrWaitGrid);
      return false;
    }
    __nanosleep(32);
  }
}

// ------------------------------------------------------------ async copies -
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tiled tensor copy global -> shared (no multicast).
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, int32_t c0,
                                            int32_t c1, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// --------------------------------------------- programmatic dependent launch
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// -------------------------------------------------------- cluster helpers -
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// ---------------------------------------------------------- warp-level MMA -
// D(16x8, f32) = A(16x16, f16, row) * B(16x8, f16, col) + C
__device__ __forceinline__ void mma_16816(float d[4], const uint32_t a[4], uint32_t b0,
                                          uint32_t b1, const float c[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

// ------------------------------------------------------------ tcgen05 ops --
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
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

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16, issued by one thread.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once all tcgen05 ops previously issued by this thread finish.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t r[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// UMMA shared-memory descriptor, K-major operand with 128-byte swizzle:
// rows of 128 B, 8-row atoms of 1024 B (stride byte offset), version 1.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);        // start address
  d |= (uint64_t)1 << 16;                             // leading byte offset (unused)
  d |= (uint64_t)(1024 >> 4) << 32;                   // stride byte offset
  d |= (uint64_t)1 << 46;                             // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                             // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: A = B = F16, D = F32, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4)                 // D format F32
         | (0u << 7) | (0u << 10)  // A, B format F16
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace dvssq
