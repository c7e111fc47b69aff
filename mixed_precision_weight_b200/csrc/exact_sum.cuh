// Exact +-1 Hadamard sums of one row-block of BF16 values, rounded once to
// fp64 (round to nearest, ties to even).
//
// The encoder rotates W by H_K = diag(H_b, ...), H_b = S_b / sqrt(b), with
// S_b Sylvester's +-1 matrix (MiniCPM5-2B-Hadamard-GSQ model card,
// "Mathematical Foundations" §1; Spark-X2.5-4B-Hadamard-GSQ model card,
// Tier B), and its codes are defined on RN64 of the EXACT sum
// sum_l S_b[j, l] w_l.  An fp64 butterfly gives that value only when every
// partial sum is exact, which holds when the block's BF16 exponents span at
// most 45 - log2(b) bits.  Blocks outside that bound are summed here in
// integers: every BF16 value is sig * 2^(o - 133) with an 8-bit significand
// and o in [0, 253], so the sum is an integer multiple of 2^-133 below
// 2^(8 + 253 + 8).  It is accumulated in eight carry-save 32-bit digits
// (int64 each, so 256 terms of at most 39 bits never overflow), normalised,
// and rounded to 53 bits with a sticky bit.
//
// Host and device code: the host build serves the CPU test of this routine.
#pragma once

#include <stdint.h>

#ifndef __CUDACC__
#define __host__
#define __device__
#define __forceinline__ inline
#endif

namespace dvssq {

__host__ __device__ __forceinline__ int clz32(uint32_t v) {
#ifdef __CUDA_ARCH__
  return __clz(v);
#else
  return v ? __builtin_clz(v) : 32;
#endif
}

__host__ __device__ __forceinline__ int parity32(uint32_t v) {
#ifdef __CUDA_ARCH__
  return __popc(v) & 1;
#else
  return __builtin_popcount(v) & 1;
#endif
}

// 2^e as a double for e in [-1022, 1023] (exact).
__host__ __device__ __forceinline__ double pow2_f64(int e) {
  const uint64_t bits = (uint64_t)(e + 1023) << 52;
#ifdef __CUDA_ARCH__
  return __longlong_as_double((long long)bits);
#else
  double d;
  static_assert(sizeof(d) == sizeof(bits), "fp64");
  __builtin_memcpy(&d, &bits, sizeof(d));
  return d;
#endif
}

// True when the row-block contains an Inf or NaN: the exact path then
// leaves the fp64 butterfly's (non-finite) result in place.
__host__ __device__ __forceinline__ bool block_has_nonfinite(const uint16_t *w, int b) {
  bool bad = false;
  for (int l = 0; l < b; ++l) bad |= ((w[l] >> 7) & 0xFFu) == 0xFFu;
  return bad;
}

// RN64( sum_l S_b[o, l] * w[l] ), S_b[o, l] = (-1)^popcount(o & l), for the
// BF16 bit patterns w[0..b) (finite).  An exact zero gives +0.0.
__host__ __device__ inline double exact_pm_sum(const uint16_t *w, int b, int o) {
  int64_t acc[8];
  for (int d = 0; d < 8; ++d) acc[d] = 0;
  for (int l = 0; l < b; ++l) {
    const uint32_t bits = w[l];
    const uint32_t e = (bits >> 7) & 0xFFu, m = bits & 0x7Fu;
    if (e == 0 && m == 0) continue;                       // +-0
    const uint32_t sig = e ? (m | 0x80u) : m;             // subnormal: m * 2^-133
    const int off = e ? (int)e - 1 : 0;                   // lsb = 2^(off - 133)
    const int64_t term = (int64_t)sig << (off & 31);      // < 2^39
    const bool neg = ((bits >> 15) ^ (uint32_t)parity32((uint32_t)(o & l))) & 1u;
    const int dg = off >> 5;                              // 0..7
    for (int d = 0; d < 8; ++d) acc[d] += (d == dg) ? (neg ? -term : term) : 0;
  }
  // normalise: digits in [0, 2^32), the sign in the final carry
  uint32_t dig[9];
  int64_t carry = 0;
  for (int d = 0; d < 8; ++d) {
    const int64_t v = acc[d] + carry;
    dig[d] = (uint32_t)(v & 0xFFFFFFFFll);
    carry = v >> 32;                                      // arithmetic shift
  }
  dig[8] = (uint32_t)(carry & 0xFFFFFFFFll);
  const bool negative = carry < 0;
  if (negative) {                                         // |N| = ~N + 1 over 288 bits
    uint64_t c = 1;
    for (int d = 0; d < 9; ++d) {
      const uint64_t v = (uint64_t)(~dig[d]) + c;
      dig[d] = (uint32_t)v;
      c = v >> 32;
    }
  }
  int h = -1;
  for (int d = 8; d >= 0; --d)
    if (h < 0 && dig[d] != 0) h = d;
  if (h < 0) return 0.0;
  // 96-bit window of digits h, h-1, h-2 (missing digits are 0), sticky below
  const uint64_t d1 = h >= 1 ? dig[h - 1] : 0, d2 = h >= 2 ? dig[h - 2] : 0;
  bool sticky = false;
  for (int d = 0; d < 9; ++d) sticky |= (d < h - 2) && dig[d] != 0;
  const uint64_t hi = dig[h];                             // bits 64..95 of the window
  const uint64_t lo = (d1 << 32) | d2;                    // bits 0..63
  const int nb = 64 + 32 - clz32(dig[h]);                 // significant bits of the window
  uint64_t mant;
  int shift = nb - 53;                                    // >= 12: nb >= 65
  {
    // mant = window >> shift; rem = low `shift` bits (shift in [12, 43])
    mant = (hi << (64 - shift)) | (lo >> shift);
    const uint64_t rem = lo & ((1ull << shift) - 1ull);
    const uint64_t half = 1ull << (shift - 1);
    const bool up = rem > half || (rem == half && (sticky || (mant & 1ull)));
    if (up) {
      ++mant;
      if (mant == (1ull << 53)) {
        mant >>= 1;
        ++shift;
      }
    }
  }
  // value = mant * 2^(shift + 32 (h - 2) - 133)
  const int e2 = shift + 32 * (h - 2) - 133;
  double r = (double)mant;                                // exact: mant < 2^53
  // |N| lies in [2^-133, 2^136], so e2 is in [-185, 84] and the product is
  // an exact normal fp64 value
  r = r * pow2_f64(e2);
  return negative ? -r : r;
}

}  // namespace dvssq
