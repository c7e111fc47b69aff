// DV-SSQ encoder kernels (Spark-X2.5-4B-Hadamard-GSQ model card, DV-SSQ
// Tiers A and B; MiniCPM5-2B-Hadamard-GSQ model card, Mathematical
// Foundations §1-§2).
//
//   pass 1  W_rot = W . H_K row-block by row-block in fp64 (exact +-1 sums,
//           one scale by 1/sqrt(b)); per-column sum of squares over fixed
//           chunks of 16 rows; exactness check of every row-block.
//   score   chunk partials summed in ascending order, score = a * sqrt(ssq).
//   select  the n_sal largest scores (ties -> lower index) by an MSB-first
//           radix select in one CTA; outputs sorted indices, a column bit
//           mask and per-32-column prefix counts.
//   pass 2  rotation again, INT4 group RTN with BF16 scales, nibble packing,
//           optional fp32 residual; salient values to an fp64 stash in the
//           workspace and their per-row maxima by atomic max.
//   pass 3  INT8 tier from the stash: one BF16 scale per row, codes.
#include <algorithm>

#include "common.cuh"
#include "fwht_group.cuh"
#include "kernels.h"

namespace dvssq {

constexpr int kSsqChunk = 16;     // rows per fixed-order partial (salience)
constexpr int kStages = 4;        // cp.async ring depth per group (row-blocks)

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// RN64(1/m) for the BF16 significands m = 128..255, filled once per device by
// the host (C double division, correctly rounded).
__constant__ double kRecipMant[128];

// RN64(1 / s) for a positive BF16 value s given by its bits: for normal s =
// m * 2^(e-7) this is RN64(1/m) * 2^(7-e), exact; other values divide.
__device__ __forceinline__ double recip_bf16(uint16_t bits) {
  const uint32_t eb = (bits >> 7) & 0xFFu;
  if (eb == 0u || eb == 0xFFu) return __ddiv_rn(1.0, bf16_bits_to_f64(bits));
  const double scale = __longlong_as_double((long long)(134 - (int)eb + 1023) << 52);
  return kRecipMant[bits & 0x7Fu] * scale;
}

// bf16_rn(RN64(a / d)) for a >= 0: the product a * RN64(1/d) is within two
// fp64 ulps of RN64(a / d); only when it lies within 8 ulps of a BF16
// rounding midpoint (or below the BF16 normal range) is the division done.
__device__ __forceinline__ uint16_t bf16_of_quotient(double a, double d, double rinv) {
  double q = __dmul_rn(a, rinv);
  const unsigned long long u = (unsigned long long)__double_as_longlong(q);
  const long long dist = (long long)(u & ((1ull << 45) - 1)) - (1ll << 44);
  if ((dist >= -8 && dist <= 8) || (q != 0.0 && q < 0x1p-120)) q = __ddiv_rn(a, d);
  return f64_to_bf16_rn(q);
}

// Exponent statistics of one thread's 16 BF16 inputs: (max biased exponent,
// min of max(biased exponent, 1)) over nonzero values.
__device__ __forceinline__ void exp_stats(const uint16_t *x, int &emax, int &emin1) {
#pragma unroll
  for (int a = 0; a < 16; ++a) {
    uint32_t m = x[a] & 0x7FFFu;
    int eb = (int)(m >> 7);
    if (m != 0) {
      emax = max(emax, eb);
      emin1 = min(emin1, max(eb, 1));
    }
  }
}

// ---------------------------------------------------------------- pass 1 --
// One group of P threads per (row chunk, column block) pair; the group walks
// the chunk's rows in ascending order so that each column's partial sum of
// squares follows the fixed order acc = acc + w*w.
template <int B>
__global__ void __launch_bounds__(128) enc_pass1_kernel(const uint16_t *__restrict__ W, int M,
                                                        int K, double c, double *__restrict__ part,
                                                        unsigned long long *__restrict__ info) {
  constexpr int P = B / 16;
  constexpr int GPW = 32 / P;
  constexpr int NG = GPW * 4;
  constexpr int SCR = GroupScratch<B>::kElems;
  __shared__ double scratch[NG][SCR];
  __shared__ __align__(16) uint16_t ring[NG][kStages][B];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = lane / P, t = lane % P;
  const int g = warp * GPW + gw;
  const int nkb = K / B;
  const int nchunk = (M + kSsqChunk - 1) / kSsqChunk;
  const long long pair = (long long)blockIdx.x * NG + g;
  const bool active = pair < (long long)nchunk * nkb;
  const int chunk = active ? (int)(pair / nkb) : 0;
  const int kb = active ? (int)(pair % nkb) : 0;
  const int r0 = chunk * kSsqChunk;
  const int nrows = active ? min(kSsqChunk, M - r0) : 0;

  // Each row-block is B*2 bytes = 2B/16 16-byte pieces; P threads copy them.
  constexpr int PIECES = B * 2 / 16;
  auto issue = [&](int i) {
    if (i < nrows) {
      const uint16_t *src = W + (size_t)(r0 + i) * K + (size_t)kb * B;
      uint16_t *dst = ring[g][i % kStages];
#pragma unroll
      for (int p = t; p < PIECES; p += P) cp_async16(dst + p * 8, src + p * 8);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) issue(i);

  double ssq[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) ssq[j] = 0.0;
  unsigned long long inexact = 0;
  const int lg = (B == 256) ? 8 : 7;

  for (int i = 0; i < kSsqChunk; ++i) {   // uniform trip count keeps the warp converged
    issue(i + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();
    uint16_t xin[16];
    const uint16_t *buf = ring[g][i % kStages];
#pragma unroll
    for (int a = 0; a < 16; ++a) xin[a] = buf[P * a + t];
    int emax = -1, emin1 = 1 << 20;
    exp_stats(xin, emax, emin1);
    double v[16];
#pragma unroll
    for (int a = 0; a < 16; ++a) v[a] = bf16_bits_to_f64(xin[a]);
    fwht_group<B>(v, scratch[g], t);
    if (i < nrows) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        // b = 256: c = 1/16 scales every square and sum exactly; apply c^2 once
        const double w = B == 256 ? v[j] : __dmul_rn(v[j], c);
        ssq[j] = __dadd_rn(ssq[j], __dmul_rn(w, w));
      }
    }
    // exactness of this row-block: reduce over the P lanes of the group
#pragma unroll
    for (int o = 1; o < P; o <<= 1) {
      emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
      emin1 = min(emin1, __shfl_xor_sync(0xffffffffu, emin1, o));
    }
    if (t == 0 && i < nrows && emax >= 0 && (emax - emin1) > 45 - lg) ++inexact;
    __syncwarp();
  }
  cp_async_wait<0>();
  if (active) {
    double *dst = part + (size_t)chunk * K + (size_t)kb * B + 16 * t;
    if (B == 256) {
      const double c2 = c * c;
#pragma unroll
      for (int j = 0; j < 16; ++j) ssq[j] = __dmul_rn(ssq[j], c2);
    }
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      double2 d = make_double2(ssq[j], ssq[j + 1]);
      *reinterpret_cast<double2 *>(dst + j) = d;
    }
    if (t == 0 && inexact) atomicAdd(&info[0], inexact);
  }
}

// ----------------------------------------------------------------- score --
// ssq_j = sum over groups (ascending) of [sum over the group's 8 chunk
// partials (ascending)]; score_j = a_j * sqrt(ssq_j).  A CTA owns 32 columns:
// its 256 threads form group sums (8 independent loads each) into shared
// memory, 64 groups at a time, and 32 threads add them in order.
constexpr int kSsqGroup = 8;
constexpr int kScoreCols = 32;
constexpr int kScoreGroupsPerPass = 64;

__global__ void __launch_bounds__(256) enc_score_kernel(
    const double *__restrict__ part, int nchunk, int K, const float *__restrict__ act_scale,
    double *__restrict__ score, unsigned long long *__restrict__ info) {
  __shared__ double gs[kScoreGroupsPerPass][kScoreCols + 1];
  const int tid = threadIdx.x, col = tid & 31, sub = tid >> 5;     // 8 sub-rows
  const int j0 = blockIdx.x * kScoreCols;
  const int j = j0 + col;
  const int ngroups = (nchunk + kSsqGroup - 1) / kSsqGroup;
  double tot = 0.0;
  for (int g0 = 0; g0 < ngroups; g0 += kScoreGroupsPerPass) {
    const int gn = min(kScoreGroupsPerPass, ngroups - g0);
    for (int gi = sub; gi < gn; gi += 8) {
      const int c0 = (g0 + gi) * kSsqGroup;
      double v[kSsqGroup];
#pragma unroll
      for (int u = 0; u < kSsqGroup; ++u)
        v[u] = (j < K && c0 + u < nchunk) ? part[(size_t)(c0 + u) * K + j] : 0.0;
      double sgrp = 0.0;
#pragma unroll
      for (int u = 0; u < kSsqGroup; ++u)
        if (c0 + u < nchunk) sgrp = __dadd_rn(sgrp, v[u]);
      gs[gi][col] = sgrp;
    }
    __syncthreads();
    if (sub == 0)
      for (int gi = 0; gi < gn; ++gi) tot = __dadd_rn(tot, gs[gi][col]);
    __syncthreads();
  }
  if (sub == 0 && j < K) {
    const double s = __dmul_rn((double)act_scale[j], __dsqrt_rn(tot));
    if (!isfinite(s)) atomicAdd(&info[2], 1ull);
    score[j] = s;
  }
}

// ---------------------------------------------------------------- select --
// Order-preserving 64-bit key of a non-NaN double (-0 treated as +0).
__device__ __forceinline__ unsigned long long order_key(double d) {
  if (d == 0.0) d = 0.0;
  const unsigned long long u = (unsigned long long)__double_as_longlong(d);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

constexpr int kSelThreads = 1024;
constexpr int kSelSmemKeys = 16384;       // keys kept in shared memory up to this K

// Exclusive prefix sum of v over the CTA in thread order (all threads call).
__device__ __forceinline__ int block_exclusive_scan(int v, int *s_warp, int *s_total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int w = lane < nw ? s_warp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < nw) s_warp[lane] = wi - w;
    if (lane == nw - 1) *s_total = wi;
  }
  __syncthreads();
  const int r = s_warp[warp] + incl - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kSelThreads) enc_select_kernel(
    const double *__restrict__ score, int K, int n_sal, int M, int32_t *__restrict__ sal_idx,
    uint32_t *__restrict__ sal_mask, int32_t *__restrict__ sal_prefix,
    unsigned long long *__restrict__ rowmax) {
  extern __shared__ unsigned long long skeys[];
  __shared__ unsigned int hist[256];
  __shared__ int s_warp[32];
  __shared__ int s_total;
  __shared__ unsigned long long s_prefix;
  __shared__ unsigned int s_krem;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool in_smem = K <= kSelSmemKeys;

  for (int i = tid; i < M; i += kSelThreads) rowmax[i] = 0ull;    // for pass 2
  for (int w = tid; w < (K + 31) / 32; w += kSelThreads) sal_mask[w] = 0u;
  if (n_sal == 0) return;
  if (in_smem)
    for (int j = tid; j < K; j += kSelThreads) skeys[j] = order_key(score[j]);
  __syncthreads();
  auto key = [&](int j) { return in_smem ? skeys[j] : order_key(score[j]); };
  // this thread's keys j = tid + 1024 i live in registers while K <= 16384
  constexpr int KPT = kSelSmemKeys / kSelThreads;
  unsigned long long rk[KPT];
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const int j = tid + i * kSelThreads;
    rk[i] = (in_smem && j < K) ? skeys[j] : 0ull;
  }
  const int iters = (K + kSelThreads - 1) / kSelThreads;

  unsigned long long prefix = 0, pmask = 0;
  unsigned int krem = (unsigned int)n_sal;
  for (int shift = 56; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    auto count = [&](unsigned long long k, int j) {
      const bool live = j < K && (k & pmask) == prefix;
      const unsigned int digit = (unsigned int)((k >> shift) & 255);
      // when every live lane has the same digit (the common case in the high
      // passes) one lane adds the count; otherwise each live lane adds one
      const unsigned int act = __ballot_sync(0xffffffffu, live);
      if (act) {
        const int leader = __ffs(act) - 1;
        const unsigned int d0 = __shfl_sync(0xffffffffu, digit, leader);
        if (__all_sync(0xffffffffu, !live || digit == d0)) {
          if (lane == leader) atomicAdd(&hist[d0], (unsigned int)__popc(act));
        } else if (live) {
          atomicAdd(&hist[digit], 1u);
        }
      }
    };
    if (in_smem) {
#pragma unroll
      for (int i = 0; i < KPT; ++i)
        if (i < iters) count(rk[i], tid + i * kSelThreads);    // uniform across the CTA
    } else {
      for (int i = 0; i < iters; ++i) {
        const int j = tid + i * kSelThreads;
        count(j < K ? key(j) : 0ull, j);
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits [8l, 8l+8); find the digit holding the krem-th largest
      unsigned int loc = 0;
#pragma unroll
      for (int d = 0; d < 8; ++d) loc += hist[8 * lane + d];
      // suffix sums over lanes, inclusive from the top digit
      unsigned int suf = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int n = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += n;
      }
      const unsigned int above = suf - loc;   // count in lanes above this one
      if (above < krem && krem <= suf) {
        unsigned int cum = above;
        int d = 8 * lane + 7;
        for (; d > 8 * lane; --d) {
          if (cum + hist[d] >= krem) break;
          cum += hist[d];
        }
        s_krem = krem - cum;
        s_prefix = prefix | ((unsigned long long)d << shift);
      }
    }
    __syncthreads();
    krem = s_krem;
    prefix = s_prefix;
    pmask |= 255ull << shift;
    __syncthreads();
  }
  // prefix = key of the n_sal-th largest score; krem = how many keys equal to
  // it are taken, lowest indices first.  Contiguous index ranges per thread.
  const int per = (K + kSelThreads - 1) / kSelThreads;
  const int j0 = min(K, tid * per), j1 = min(K, j0 + per);
  int n_eq = 0;
  for (int j = j0; j < j1; ++j) n_eq += key(j) == prefix;
  const int eq_before = block_exclusive_scan(n_eq, s_warp, &s_total);
  int n_sel = 0;
  {
    int eqr = eq_before;
    for (int j = j0; j < j1; ++j) {
      const unsigned long long k = key(j);
      n_sel += k > prefix || (k == prefix && (unsigned)(eqr++) < krem);
    }
  }
  int pos = block_exclusive_scan(n_sel, s_warp, &s_total);
  int eqr = eq_before;
  for (int j = j0; j < j1; ++j) {
    const unsigned long long k = key(j);
    const bool sel = k > prefix || (k == prefix && (unsigned)(eqr++) < krem);
    if ((j & 31) == 0) sal_prefix[j >> 5] = pos;
    if (sel && pos < n_sal) {
      sal_idx[pos++] = j;
      atomicOr(&sal_mask[j >> 5], 1u << (j & 31));
    }
  }
}

// ---------------------------------------------------------------- pass 2 --
// One group of P threads per (8 rows, column block): rotate again, INT4 group
// RTN with BF16 scales, nibble packing, optional fp32 residual.  Salient
// values go to the fp64 stash sv[row][entry] and the row maxima of their
// magnitudes to rowmax (atomic max on the bit patterns of non-negative
// doubles).  For b = 256 the scale c = 1/16 is a power of two: the stash and
// rowmax hold the unscaled sums and pass 3 applies c exactly, and the codes
// use w * inv = v * (c * inv) exactly.
constexpr int kP2Rows = 8;

template <int B, bool RESID>
__global__ void __launch_bounds__(128) enc_pass2_kernel(
    const uint16_t *__restrict__ W, int M, int K, int n_sal, double c,
    const uint32_t *__restrict__ sal_mask, const int32_t *__restrict__ sal_prefix,
    uint8_t *__restrict__ q4, uint16_t *__restrict__ s4, double *__restrict__ sv,
    unsigned long long *__restrict__ rowmax, float *__restrict__ resid,
    unsigned long long *__restrict__ info) {
  constexpr int P = B / 16;
  constexpr int GPW = 32 / P;
  constexpr int NG = GPW * 4;
  constexpr int SCR = GroupScratch<B>::kElems;
  constexpr bool kPow2 = B == 256;
  __shared__ double scratch[NG][SCR];
  __shared__ __align__(16) uint16_t ring[NG][kStages][B];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = lane / P, t = lane % P;
  const int g = warp * GPW + gw;
  const int nkb = K / B;
  const int nrc = (M + kP2Rows - 1) / kP2Rows;
  const long long pair = (long long)blockIdx.x * NG + g;
  const bool active = pair < (long long)nrc * nkb;
  const int rc = active ? (int)(pair / nkb) : 0;
  const int kb = active ? (int)(pair % nkb) : 0;
  const int r0 = rc * kP2Rows;
  const int nrows = active ? min(kP2Rows, M - r0) : 0;
  const double kInv7 = 1.0 / 7.0;

  // salient columns among this thread's 16 are the same for every row
  const int col0 = kb * B + 16 * t;
  const uint32_t mword = sal_mask[col0 >> 5];
  const int bit0 = col0 & 31;
  const uint32_t m16 = (mword >> bit0) & 0xFFFFu;
  const int ebase = m16 ? sal_prefix[col0 >> 5] + __popc(mword & ((1u << bit0) - 1u)) : 0;

  constexpr int PIECES = B * 2 / 16;
  auto issue = [&](int i) {
    if (i < nrows) {
      const uint16_t *src = W + (size_t)(r0 + i) * K + (size_t)kb * B;
      uint16_t *dst = ring[g][i % kStages];
#pragma unroll
      for (int p = t; p < PIECES; p += P) cp_async16(dst + p * 8, src + p * 8);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) issue(i);

  unsigned long long unsafe = 0;
  for (int i = 0; i < kP2Rows; ++i) {
    issue(i + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();
    double v[16];
    const uint16_t *buf = ring[g][i % kStages];
#pragma unroll
    for (int a = 0; a < 16; ++a) v[a] = bf16_bits_to_f64(buf[P * a + t]);
    fwht_group<B>(v, scratch[g], t);
    const int row = r0 + i;
    // v holds the values the codes see: unscaled sums (b = 256) or w = c * sum
    if (!kPow2) {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __dmul_rn(v[j], c);
    }
    double amax = 0.0, amax8 = 0.0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if ((m16 >> j) & 1u) amax8 = fmax(amax8, fabs(v[j]));
      else amax = fmax(amax, fabs(v[j]));
    }
    amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, 1));   // 64-column group
    amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
#pragma unroll
    for (int o = 1; o < P; o <<= 1) amax8 = fmax(amax8, __shfl_xor_sync(0xffffffffu, amax8, o));
    // absmax of w = c * amax (exact for b = 256)
    const uint16_t sbits = bf16_of_quotient(kPow2 ? amax * c : amax, 7.0, kInv7);
    const double s = bf16_bits_to_f64(sbits);
    const double inv = s > 0.0 ? recip_bf16(sbits) : 0.0;
    const double vinv = kPow2 ? inv * c : inv;    // multiplies v
    uint32_t word[2] = {0u, 0u};
    int e = ebase;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      int q = 0;
      if (!((m16 >> j) & 1u)) {
        q = __double2int_rn(__dmul_rn(v[j], vinv));
        q = min(7, max(-8, q));
      } else {
        if (i < nrows && e < n_sal) sv[(size_t)row * n_sal + e] = v[j];
        ++e;
      }
      word[j >> 3] |= ((uint32_t)q & 0xFu) << (4 * (j & 7));
    }
    if (i < nrows) {
      *reinterpret_cast<uint2 *>(q4 + (size_t)row * (K / 2) + (col0 >> 1)) =
          make_uint2(word[0], word[1]);
      if ((t & 3) == 0) {
        s4[(size_t)row * (K / 64) + (col0 >> 6)] = sbits;
        if (s > 0.0 && (s < 0x1p-17 || s > 8188.0)) ++unsafe;
      }
      if (t == 0 && amax8 > 0.0)
        atomicMax(&rowmax[row], (unsigned long long)__double_as_longlong(amax8));
      if (RESID) {
        float rres[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const double w = kPow2 ? v[j] * c : v[j];
          if ((m16 >> j) & 1u) {
            rres[j] = 0.0f;
          } else {
            const int q = (int)((word[j >> 3] >> (4 * (j & 7))) << 28) >> 28;
            rres[j] = (float)__dsub_rn(w, (double)q * s);
          }
        }
        float4 *dst = reinterpret_cast<float4 *>(resid + (size_t)row * K + col0);
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          dst[j / 4] = make_float4(rres[j], rres[j + 1], rres[j + 2], rres[j + 3]);
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  if (active && unsafe) atomicAdd(&info[1], unsafe);
}

// ---------------------------------------------------------------- pass 3 --
// INT8 tier: s8 = bf16_rn(max|w| / 127), q8 = clip(rint(w * (1/s8))).  The
// stash holds w / vscale (vscale = c for b = 256, else 1).  One thread per 8
// entries of a row.
__global__ void __launch_bounds__(256) enc_pass3_kernel(
    const double *__restrict__ sv, const unsigned long long *__restrict__ rowmax, int M,
    int n_sal, double vscale, int8_t *__restrict__ q8, uint16_t *__restrict__ s8,
    unsigned long long *__restrict__ info) {
  const int n8 = n_sal / 8;
  const long long items = n8 > 0 ? (long long)M * n8 : (long long)M;
  const double kInv127 = 1.0 / 127.0;
  for (long long it = (long long)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (long long)gridDim.x * blockDim.x) {
    const int row = n8 > 0 ? (int)(it / n8) : (int)it;
    const int e0 = n8 > 0 ? 8 * (int)(it % n8) : 0;
    const double2 *src = reinterpret_cast<const double2 *>(sv + (size_t)row * n_sal + e0);
    double2 d[4];
    if (n8 > 0) {
#pragma unroll
      for (int u = 0; u < 4; ++u) d[u] = src[u];
    }
    const double m = __longlong_as_double((long long)rowmax[row]) * vscale;
    const uint16_t sbits = bf16_of_quotient(m, 127.0, kInv127);
    const double sv8 = bf16_bits_to_f64(sbits);
    if (e0 == 0) {
      s8[row] = sbits;
      if (sv8 > 0.0 && (sv8 < 0x1p-17 || sv8 > 511.0)) atomicAdd(&info[1], 1ull);
    }
    if (n8 == 0) continue;
    const double vinv = sv8 > 0.0 ? recip_bf16(sbits) * vscale : 0.0;
    uint32_t pk[2] = {0u, 0u};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int qa = __double2int_rn(__dmul_rn(d[u].x, vinv));
      int qb = __double2int_rn(__dmul_rn(d[u].y, vinv));
      qa = min(127, max(-128, qa));
      qb = min(127, max(-128, qb));
      pk[u >> 1] |= (((uint32_t)qa & 0xFFu) | (((uint32_t)qb & 0xFFu) << 8)) << (16 * (u & 1));
    }
    *reinterpret_cast<uint2 *>(q8 + (size_t)row * n_sal + e0) = make_uint2(pk[0], pk[1]);
  }
}

// --------------------------------------------------------------- launch ---
namespace {
struct EncodeLayout {
  size_t info, part, score, mask, pref, rowmax, sv, total;
};
EncodeLayout encode_layout(int M, int K, int n_sal) {
  const size_t nchunk = (size_t)(M + kSsqChunk - 1) / kSsqChunk;
  EncodeLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  L.info = take(4 * sizeof(unsigned long long));
  L.part = take(nchunk * (size_t)K * sizeof(double));
  L.score = take((size_t)K * sizeof(double));
  L.mask = take((size_t)((K + 31) / 32) * sizeof(uint32_t));
  L.pref = take((size_t)((K + 31) / 32) * sizeof(int32_t));
  L.rowmax = take((size_t)M * sizeof(unsigned long long));
  L.sv = take((size_t)M * n_sal * sizeof(double));
  L.total = off;
  return L;
}
}  // namespace

size_t encode_workspace_bytes(int M, int K, int n_sal) { return encode_layout(M, K, n_sal).total; }

cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t st, Launcher &L) {
  const int M = a.M, K = a.K, B = a.block;
  const int nchunk = (M + kSsqChunk - 1) / kSsqChunk;
  const EncodeLayout lay = encode_layout(M, K, a.n_sal);
  char *ws = static_cast<char *>(a.workspace);
  auto *info = reinterpret_cast<unsigned long long *>(ws + lay.info);
  auto *part = reinterpret_cast<double *>(ws + lay.part);
  auto *score = reinterpret_cast<double *>(ws + lay.score);
  auto *mask = reinterpret_cast<uint32_t *>(ws + lay.mask);
  auto *pref = reinterpret_cast<int32_t *>(ws + lay.pref);
  auto *rowmax = reinterpret_cast<unsigned long long *>(ws + lay.rowmax);
  auto *sv = reinterpret_cast<double *>(ws + lay.sv);
  const double c = sqrt(1.0 / (double)B);

  cudaError_t e = cudaMemsetAsync(info, 0, 4 * sizeof(unsigned long long), st);
  if (e != cudaSuccess) return e;
  const int nkb = K / B;
  const int P = B / 16, NG = (32 / P) * 4;
  const long long pairs1 = (long long)nchunk * nkb;
  dim3 g1((unsigned)((pairs1 + NG - 1) / NG));
  if (B == 256)
    e = L.launch("enc_pass1", enc_pass1_kernel<256>, g1, dim3(128), 0, st, false,
                 (const uint16_t *)a.W, M, K, c, part, info);
  else
    e = L.launch("enc_pass1", enc_pass1_kernel<128>, g1, dim3(128), 0, st, false,
                 (const uint16_t *)a.W, M, K, c, part, info);
  if (e != cudaSuccess) return e;
  e = L.launch("enc_score", enc_score_kernel, dim3((K + kScoreCols - 1) / kScoreCols), dim3(256),
               0, st, false,
               (const double *)part, nchunk, K, a.act_scale, score, info);
  if (e != cudaSuccess) return e;
  const size_t sel_smem = K <= kSelSmemKeys ? (size_t)K * sizeof(unsigned long long) : 0;
  e = L.launch("enc_select", enc_select_kernel, dim3(1), dim3(kSelThreads), sel_smem, st, false,
               (const double *)score, K, a.n_sal, M, a.sal_idx, mask, pref, rowmax);
  if (e != cudaSuccess) return e;
  const long long pairs2 = (long long)((M + kP2Rows - 1) / kP2Rows) * nkb;
  dim3 g2((unsigned)((pairs2 + NG - 1) / NG));
#define DVSSQ_PASS2(BB, RR)                                                                  \
  L.launch("enc_pass2", enc_pass2_kernel<BB, RR>, g2, dim3(128), 0, st, false,            \
           (const uint16_t *)a.W, M, K, a.n_sal, c, (const uint32_t *)mask,               \
           (const int32_t *)pref, a.q4, a.s4, sv, rowmax, a.resid, info)
  if (B == 256)
    e = a.resid ? DVSSQ_PASS2(256, true) : DVSSQ_PASS2(256, false);
  else
    e = a.resid ? DVSSQ_PASS2(128, true) : DVSSQ_PASS2(128, false);
#undef DVSSQ_PASS2
  if (e != cudaSuccess) return e;
  const long long items = a.n_sal > 0 ? (long long)M * (a.n_sal / 8) : (long long)M;
  const long long g3 = std::min<long long>((items + 255) / 256, 148LL * 16);
  const double vscale = B == 256 ? c : 1.0;
  e = L.launch("enc_pass3", enc_pass3_kernel, dim3((unsigned)g3), dim3(256), 0, st, false,
               (const double *)sv, (const unsigned long long *)rowmax, M, a.n_sal, vscale, a.q8,
               a.s8, info);
  if (e != cudaSuccess) return e;
  if (a.info_host != nullptr) {
    unsigned long long h[4];
    e = cudaMemcpyAsync(h, info, sizeof(h), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    a.info_host[0] = (int64_t)h[0];
    a.info_host[1] = (int64_t)h[1];
    a.info_host[2] = (int64_t)h[2];
  }
  return cudaSuccess;
}

cudaError_t prepare_encode_kernels() {
  cudaError_t e;
  for (const void *f :
       {(const void *)enc_pass1_kernel<256>, (const void *)enc_pass1_kernel<128>,
        (const void *)enc_pass2_kernel<256, false>, (const void *)enc_pass2_kernel<128, false>,
        (const void *)enc_pass2_kernel<256, true>, (const void *)enc_pass2_kernel<128, true>})
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
  double recip[128];
  for (int m = 0; m < 128; ++m) recip[m] = 1.0 / (double)(128 + m);
  if ((e = cudaMemcpyToSymbol(kRecipMant, recip, sizeof(recip))) != cudaSuccess) return e;
  return cudaFuncSetAttribute(enc_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kSelSmemKeys * (int)sizeof(unsigned long long));
}

}  // namespace dvssq
