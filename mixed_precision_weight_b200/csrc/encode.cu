// DV-SSQ encoder kernels (Spark-X2.5-4B-Hadamard-GSQ model card, DV-SSQ
// Tiers A and B; MiniCPM5-2B-Hadamard-GSQ model card, Mathematical
// Foundations §1-§2).
//
//   pass 1  W_rot = W . H_K row-block by row-block in fp64 (exact +-1 sums,
//           one scale by 1/sqrt(b)); per-column sums of squares over fixed
//           chunks of 16 rows, summed by the CTA into groups of 8 chunks; the
//           last CTA of each column block adds the groups in order and writes
//           score = a * sqrt(ssq).  Every chunk is tested for exact fp64
//           summation; a chunk that fails is recomputed row by row, its
//           flagged row-blocks summed exactly in integers (exact_sum.cuh),
//           and a per-(chunk, column block) row mask is written for pass 2.
//   select  the n_sal largest scores (ties -> lower index) by an MSB-first
//           radix select in one CTA that stops as soon as the boundary digit
//           is taken whole; outputs sorted indices and per-32-column prefix
//           counts.
//   pass 2  whole rows per CTA (dynamic tile order): rotation again, salient
//           values (exact sums for the row-blocks pass 1 flagged) moved to a
//           shared-memory stash and zeroed in place, INT4
//           group RTN with BF16 scales, nibble packing, optional fp32
//           residual; then the INT8 tier of the CTA's rows from the stash.
#include <algorithm>

#include "common.cuh"
#include "exact_sum.cuh"
#include "fwht_group.cuh"
#include "kernels.h"

namespace dvssq {

constexpr int kSsqChunk = 16;     // rows per fixed-order partial (salience)
constexpr int kSsqGroup = 8;      // chunk partials per group sum
constexpr int kStages = 4;        // cp.async ring depth per group (row-blocks), pass 1
constexpr int kP2Stages = 3;      // the same for pass 2 (fewer: five CTAs per SM fit)
constexpr int kTileRowsMax = 64;  // rows per pass-2 tile, upper bound
constexpr int kStashSmemMax = 96 * 1024;

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

// Thread t's 16 outputs 16t .. 16t+15 of the exact +-1 sums of a row-block,
// written to out[16t + j] (rare path: out of line, and through memory, so
// that nothing of the caller's stays live across it).
__device__ __noinline__ void exact_pm_sums16(const uint16_t *w, int b, int t, double *out) {
  for (int j = 0; j < 16; ++j) out[16 * t + j] = exact_pm_sum(w, b, 16 * t + j);
}

// Per-halfword unsigned max / min of two pairs of 16-bit lanes.
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t vmin_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Exponent statistics of BF16 pairs for the exact-sum test.  Per 16-bit lane:
//   mx = max magnitude (the 15 bits below the sign),
//   mn = min over nonzero values of (magnitude - 1); a zero maps to 0xFFFF.
// Forcing the sign bits on makes every lane >= 0x8000, so subtracting one
// from each lane never borrows across the halves.
__device__ __forceinline__ void exp_pair_stats(uint32_t w, uint32_t &mx, uint32_t &mn) {
  mx = vmax_u16x2(mx, w & 0x7FFF7FFFu);
  mn = vmin_u16x2(mn, ((w | 0x80008000u) - 0x00010001u) ^ 0x80008000u);
}

// Spread test of one row-block from its (emax, emin1) over nonzero values,
// biased BF16 exponents with subnormals counted as 1: every +-1 partial sum
// of b terms is exact in fp64 when emax - emin1 <= 45 - log2(b).
__device__ __forceinline__ bool spread_exceeds(int emax, int emin1, int lg) {
  return emax >= 0 && emin1 <= 255 && (emax - emin1) > 45 - lg;
}

// ---------------------------------------------------------------- pass 1 --
// A CTA holds NG groups of P threads; group g owns the 16-row chunk
// cg * NG + g of column block kb and walks it in ascending row order, so that
// each column's chunk partial follows the fixed order acc = acc + w*w.  The
// CTA then forms the 8-chunk group sums (ascending chunks, from 0.0) in shared
// memory, and the CTA that finishes a column block last adds that block's
// group sums in ascending order and writes the scores.
// Every chunk is tested for exact fp64 summation (BF16 exponent spread of the
// whole chunk).  A chunk that fails is summed again row by row: a row whose
// own spread exceeds the bound takes the exact integer sums, and its bit is
// set in xmask[chunk * nkb + kb] (written for every chunk, 0 when it passes)
// so that pass 2 takes the same path for that row-block.
template <int B>
__global__ void __launch_bounds__(128, 6) enc_pass1_kernel(
    const uint16_t *__restrict__ W, int M, int K, double c, const float *__restrict__ act_scale,
    double *__restrict__ gpart, double *__restrict__ score, unsigned int *__restrict__ done,
    unsigned long long *__restrict__ info, uint16_t *__restrict__ xmask) {
  constexpr int P = B / 16;
  constexpr int GPW = 32 / P;
  constexpr int NG = GPW * 4;
  constexpr int SCR = GroupScratch<B>::kElems;
  static_assert(SCR >= B, "chunk partials reuse the transpose scratch");
  static_assert(NG % kSsqGroup == 0, "whole chunk groups per CTA");
  constexpr int SGC = NG / kSsqGroup;
  __shared__ double scratch[NG][SCR];
  __shared__ __align__(16) uint16_t ring[NG][kStages][B];
  __shared__ unsigned int s_last;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = lane / P, t = lane % P;
  const int g = warp * GPW + gw;
  const int nkb = K / B;
  const int nchunk = (M + kSsqChunk - 1) / kSsqChunk;
  const int nsg = (nchunk + kSsqGroup - 1) / kSsqGroup;
  const int ncg = (nchunk + NG - 1) / NG;
  const int cg = blockIdx.x / nkb, kb = blockIdx.x - cg * nkb;
  const int chunk = cg * NG + g;
  const int r0 = chunk * kSsqChunk;
  const int nrows = chunk < nchunk ? min(kSsqChunk, M - r0) : 0;
  const int lg = (B == 256) ? 8 : 7;

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
  uint32_t mx = 0u, mn = 0xFFFFFFFFu;

  for (int i = 0; i < kSsqChunk; ++i) {   // uniform trip count keeps the warp converged
    issue(i + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const uint16_t *buf = ring[g][i % kStages];
    if (i < nrows) {
      // this thread's 32 contiguous bytes of the row-block, for the exact-sum test
      const uint4 *wq = reinterpret_cast<const uint4 *>(buf) + 2 * t;
      const uint4 a = wq[0], b = wq[1];
      exp_pair_stats(a.x, mx, mn); exp_pair_stats(a.y, mx, mn);
      exp_pair_stats(a.z, mx, mn); exp_pair_stats(a.w, mx, mn);
      exp_pair_stats(b.x, mx, mn); exp_pair_stats(b.y, mx, mn);
      exp_pair_stats(b.z, mx, mn); exp_pair_stats(b.w, mx, mn);
    }
    double v[16];
#pragma unroll
    for (int a = 0; a < 16; ++a) v[a] = bf16_bits_to_f64(buf[P * a + t]);
    fwht_group<B>(v, scratch[g], t);
    if (i < nrows) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        // b = 256: c = 1/16 scales every square and sum exactly; apply c^2 once
        const double w = B == 256 ? v[j] : __dmul_rn(v[j], c);
        ssq[j] = __dadd_rn(ssq[j], __dmul_rn(w, w));
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();

  // Exact-sum test, first over the whole chunk: the chunk's spread bounds the
  // spread of each of its row-blocks.  Only a chunk that fails it is summed
  // again row by row.
  {
    const uint32_t mxh = max(mx & 0xFFFFu, mx >> 16), mnh = min(mn & 0xFFFFu, mn >> 16);
    const int emax = (int)(mxh >> 7);
    const int emin1 = mnh == 0xFFFFu ? 0xFFFF : max((int)((mnh + 1u) >> 7), 1);
    // one u16x2 word reduced by max: (emax, 0xFFFF - emin1)
    uint32_t pk = ((uint32_t)emax << 16) | (uint32_t)(0xFFFF - emin1);
#pragma unroll
    for (int o = 1; o < P; o <<= 1) pk = vmax_u16x2(pk, __shfl_xor_sync(0xffffffffu, pk, o));
    const int gmax = (int)(pk >> 16), gmin1 = 0xFFFF - (int)(pk & 0xFFFFu);
    const bool fail = nrows > 0 && spread_exceeds(gmax, gmin1, lg);
    uint32_t rowmask = 0u;
    // the warp's groups may differ: the whole warp runs the row loop (its
    // shuffles and the rotation need every lane), each group keeping only
    // its own rows
    if (__any_sync(0xffffffffu, fail)) {
      unsigned long long inexact = 0;
      // a failing group sums its chunk again from zero; the other groups of
      // the warp keep theirs (their rows are not re-added)
      if (fail) {
#pragma unroll
        for (int j = 0; j < 16; ++j) ssq[j] = 0.0;
      }
      uint16_t *buf = ring[g][0];
      for (int i = 0; i < kSsqChunk; ++i) {
        const bool row = fail && i < nrows;
        if (row) {
          const uint4 *src =
              reinterpret_cast<const uint4 *>(W + (size_t)(r0 + i) * K + (size_t)kb * B);
          for (int q = t; q < B / 8; q += P) reinterpret_cast<uint4 *>(buf)[q] = src[q];
        }
        __syncwarp();
        uint32_t rx = 0u, rn = 0xFFFFFFFFu;
        if (row)
          for (int q = t; q < B / 2; q += P)
            exp_pair_stats(reinterpret_cast<const uint32_t *>(buf)[q], rx, rn);
        const uint32_t rxh = max(rx & 0xFFFFu, rx >> 16), rnh = min(rn & 0xFFFFu, rn >> 16);
        const int re = (int)(rxh >> 7);
        const int rm = rnh == 0xFFFFu ? 0xFFFF : max((int)((rnh + 1u) >> 7), 1);
        uint32_t rp = ((uint32_t)re << 16) | (uint32_t)(0xFFFF - rm);
#pragma unroll
        for (int o = 1; o < P; o <<= 1) rp = vmax_u16x2(rp, __shfl_xor_sync(0xffffffffu, rp, o));
        const bool exact_row =
            row && spread_exceeds((int)(rp >> 16), 0xFFFF - (int)(rp & 0xFFFFu), lg);
        double v[16];
#pragma unroll
        for (int a = 0; a < 16; ++a) v[a] = bf16_bits_to_f64(buf[P * a + t]);
        fwht_group<B>(v, scratch[g], t);
        if (exact_row && !block_has_nonfinite(buf, B)) {
          exact_pm_sums16(buf, B, t, scratch[g]);   // the transpose scratch is free here
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = scratch[g][16 * t + j];
        }
        if (row) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const double w = B == 256 ? v[j] : __dmul_rn(v[j], c);
            ssq[j] = __dadd_rn(ssq[j], __dmul_rn(w, w));
          }
        }
        rowmask |= (uint32_t)exact_row << i;
        inexact += exact_row;
        __syncwarp();
      }
      if (t == 0 && inexact) atomicAdd(&info[0], inexact);
    }
    if (t == 0 && chunk < nchunk) xmask[(size_t)chunk * nkb + kb] = (uint16_t)rowmask;
  }

  // chunk partials -> shared memory (the transpose scratch is free now)
  if (B == 256) {
    const double c2 = c * c;
#pragma unroll
    for (int j = 0; j < 16; ++j) ssq[j] = __dmul_rn(ssq[j], c2);
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) scratch[g][16 * t + j] = ssq[j];
  __syncthreads();
  // group sums: SGC chunk groups x B columns, two per thread
  for (int it = threadIdx.x; it < SGC * B; it += blockDim.x) {
    const int sl = it / B, col = it - sl * B;
    const int sg = cg * SGC + sl;
    if (sg >= nsg) continue;
    double s = 0.0;
#pragma unroll
    for (int u = 0; u < kSsqGroup; ++u) {
      const int gg = sl * kSsqGroup + u;
      if (cg * NG + gg < nchunk) s = __dadd_rn(s, scratch[gg][col]);
    }
    gpart[(size_t)sg * K + (size_t)kb * B + col] = s;
  }
  // the last CTA of this column block adds its group sums in order
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&done[kb], 1u) == (unsigned int)(ncg - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  unsigned long long bad = 0;
  // CPT columns per thread, their loads in flight together (10 group sums
  // of each column per batch, within pass 1's register budget); each
  // column's adds stay in ascending order
  constexpr int CPT = B / 128;
  static_assert(CPT * 128 == B, "pass 1 runs 128 threads");
  const float *as = act_scale + (size_t)kb * B + threadIdx.x;
  float a[CPT];
#pragma unroll
  for (int c2 = 0; c2 < CPT; ++c2) a[c2] = as[128 * c2];
  double tot[CPT];
#pragma unroll
  for (int c2 = 0; c2 < CPT; ++c2) tot[c2] = 0.0;
  const double *gp = gpart + (size_t)kb * B + threadIdx.x;
  for (int sg0 = 0; sg0 < nsg; sg0 += 10) {
    double gv[CPT][10];
#pragma unroll
    for (int c2 = 0; c2 < CPT; ++c2)
#pragma unroll
      for (int u = 0; u < 10; ++u)
        gv[c2][u] = sg0 + u < nsg ? __ldcg(gp + (size_t)(sg0 + u) * K + 128 * c2) : 0.0;
#pragma unroll
    for (int c2 = 0; c2 < CPT; ++c2)
#pragma unroll
      for (int u = 0; u < 10; ++u)
        if (sg0 + u < nsg) tot[c2] = __dadd_rn(tot[c2], gv[c2][u]);
  }
#pragma unroll
  for (int c2 = 0; c2 < CPT; ++c2) {
    const double s = __dmul_rn((double)a[c2], __dsqrt_rn(tot[c2]));
    bad += !isfinite(s);
    score[(size_t)kb * B + threadIdx.x + 128 * c2] = s;
  }
  if (bad) atomicAdd(&info[2], bad);
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

// MSB-first radix select over 8-bit digits.  After each digit the CTA knows
// the prefix of the n_sal-th largest key and how many keys sharing that prefix
// are still to be taken (krem).  When krem equals the number of keys with the
// prefix, every one of them is taken and the lower digits no longer matter:
// the loop stops there (typically after the exponent and two or three
// significand digits) instead of running all eight digits.
__global__ void __launch_bounds__(kSelThreads) enc_select_kernel(
    const double *__restrict__ score, int K, int n_sal, int32_t *__restrict__ sal_idx,
    int32_t *__restrict__ sal_prefix) {
  extern __shared__ unsigned long long skeys[];
  __shared__ unsigned int hist[256];
  __shared__ int s_warp[32];
  __shared__ int s_total;
  __shared__ unsigned long long s_prefix;
  __shared__ unsigned int s_krem, s_whole;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool in_smem = K <= kSelSmemKeys;
  // launched with programmatic dependent launch: the scores come from pass 1;
  // pass 2 may start its salient-independent prologue now
  pdl_wait();
  pdl_launch_dependents();

  if (n_sal == 0) {
    for (int w = tid; w < (K + 31) / 32; w += kSelThreads) sal_prefix[w] = 0;
    return;
  }
  // this thread's keys j = tid + 1024 i live in registers while K <= 16384
  // (all loads issued together), and in shared memory for the index-order
  // passes at the end
  constexpr int KPT = kSelSmemKeys / kSelThreads;
  unsigned long long rk[KPT];
  double sv[KPT];
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const int j = tid + i * kSelThreads;
    sv[i] = (in_smem && j < K) ? __ldcg(score + j) : 0.0;
  }
  unsigned long long kmax = 0ull, kmin = ~0ull;
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const int j = tid + i * kSelThreads;
    rk[i] = (in_smem && j < K) ? order_key(sv[i]) : 0ull;
    if (in_smem && j < K) {
      skeys[j] = rk[i];
      kmax = max(kmax, rk[i]);
      kmin = min(kmin, rk[i]);
    }
  }
  auto key = [&](int j) { return in_smem ? skeys[j] : order_key(score[j]); };
  const int iters = (K + kSelThreads - 1) / kSelThreads;
  if (!in_smem)
    for (int j = tid; j < K; j += kSelThreads) {
      const unsigned long long k = key(j);
      kmax = max(kmax, k);
      kmin = min(kmin, k);
    }
  // the high bits every key shares need no radix pass: start at the 8-bit
  // digit that holds the highest bit where the largest and smallest keys differ
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
  }
  __shared__ unsigned long long s_kmax[32], s_kmin[32];
  if (lane == 0) {
    s_kmax[warp] = kmax;
    s_kmin[warp] = kmin;
  }
  __syncthreads();
  if (warp == 0) {
    kmax = s_kmax[lane];
    kmin = s_kmin[lane];
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    }
    if (lane == 0) {
      s_kmax[0] = kmax;
      s_kmin[0] = kmin;
    }
  }
  __syncthreads();
  const unsigned long long diff = s_kmax[0] ^ s_kmin[0];
  const int hb = diff ? 63 - __clzll((long long)diff) : 0;      // highest differing bit
  const int top = (hb / 8) * 8;                                  // its digit's shift
  unsigned long long pmask = top >= 56 ? 0ull : ~((1ull << (top + 8)) - 1ull);
  unsigned long long prefix = s_kmax[0] & pmask;
  unsigned int krem = (unsigned int)n_sal;
  for (int shift = top; shift >= 0; shift -= 8) {
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
        s_whole = (krem - cum) == hist[d];
        s_prefix = prefix | ((unsigned long long)d << shift);
      }
    }
    __syncthreads();
    krem = s_krem;
    prefix = s_prefix;
    pmask |= 255ull << shift;
    const bool whole = s_whole;
    __syncthreads();
    if (whole) break;
  }
  // Selected: (key & pmask) > prefix, or == prefix among the first krem such
  // keys in index order.  Contiguous index ranges per thread; sal_prefix[w] is
// the number of selected columns below column 32 w.
  const int per = (K + kSelThreads - 1) / kSelThreads;
  const int j0 = min(K, tid * per), j1 = min(K, j0 + per);
  int n_eq = 0;
  for (int j = j0; j < j1; ++j) n_eq += (key(j) & pmask) == prefix;
  const int eq_before = block_exclusive_scan(n_eq, s_warp, &s_total);
  int n_sel = 0;
  {
    int eqr = eq_before;
    for (int j = j0; j < j1; ++j) {
      const unsigned long long k = key(j) & pmask;
      n_sel += k > prefix || (k == prefix && (unsigned)(eqr++) < krem);
    }
  }
  int pos = block_exclusive_scan(n_sel, s_warp, &s_total);
  int eqr = eq_before;
  for (int j = j0; j < j1; ++j) {
    const unsigned long long k = key(j) & pmask;
    const bool sel = k > prefix || (k == prefix && (unsigned)(eqr++) < krem);
    if ((j & 31) == 0) sal_prefix[j >> 5] = pos;
    if (sel && pos < n_sal) sal_idx[pos++] = j;
  }
}

// ---------------------------------------------------------------- pass 2 --
// A CTA takes tiles of R whole rows from a global counter.  Within a tile the
// R * nkb row-blocks are ordered column-block-major and split into NG equal
// runs of ipg >= kP2Stages - 1 row-blocks, one run per group, so a group's
// cp.async ring can run ahead into the next tile (whose index is fetched one
// tile early).  Per row-block the group rotates again, stages its outputs in
// shared memory, moves the block's salient values to the stash and zeroes
// them in place (so the INT4 tier needs no column mask: a zero has code 0),
// then quantises.  When the tile is done the CTA forms each row's INT8 scale
// from the stash and writes the INT8 codes.  For b = 256 the scale c = 1/16 is
// a power of two: the stash holds the unscaled sums and c is applied exactly
// in the scales, and the codes use w * inv = v * (c * inv) exactly.
struct Pass2Params {
  const uint16_t *W;
  int M, K, n_sal;
  int R, rshift;      // rows per tile (a power of two) and its log2
  int ipg;            // row-blocks per group and tile
  int ntiles;
  int stash_smem;     // 1: stash in dynamic shared memory [R][n_sal]; 0: in sv [M][n_sal]
  double c;
  const int32_t *sal_idx, *sal_prefix;
  uint8_t *q4;
  uint16_t *s4;
  int8_t *q8;
  uint16_t *s8;
  float *resid;
  double *sv;
  unsigned int *tile_ctr;
  unsigned long long *info;
  const uint16_t *xmask;   // pass 1's rows whose row-block takes the exact sums
};

// Staged outputs: thread t's 16 values at [16 t, 16 t + 16), the 16-byte
// pair m at pair position m ^ (t & 7), so that the eight threads of a
// quarter-warp store to distinct banks.
__device__ __forceinline__ int stage_pos(int col) {
  const int t = col >> 4, j = col & 15;
  return 16 * t + 2 * ((j >> 1) ^ (t & 7)) + (j & 1);
}

// Eight 4-bit codes (two's complement in the low bits of l[0..7]) into one
// word, code 2m in the low nibble of byte m.
__device__ __forceinline__ uint32_t pack_nibbles8(const uint32_t *l) {
  const uint32_t e = __byte_perm(__byte_perm(l[0], l[2], 0x0040), __byte_perm(l[4], l[6], 0x4000),
                                 0x7610);
  const uint32_t o = __byte_perm(__byte_perm(l[1], l[3], 0x0040), __byte_perm(l[5], l[7], 0x4000),
                                 0x7610);
  return (e & 0x0F0F0F0Fu) | ((o << 4) & 0xF0F0F0F0u);
}

template <int B, bool RESID>
__global__ void __launch_bounds__(128, 5) enc_pass2_kernel(const Pass2Params p) {
  constexpr int P = B / 16;
  constexpr int GPW = 32 / P;
  constexpr int NG = GPW * 4;
  constexpr int SCR0 = GroupScratch<B>::kElems;
  constexpr int SCR1 = 16 * P;
  constexpr int SCR = ((SCR0 > SCR1 ? SCR0 : SCR1) + 1) & ~1;   // even: 16-byte aligned rows
  constexpr bool kPow2 = B == 256;
  constexpr int PIECES = B * 2 / 16;
  __shared__ __align__(16) double scratch[NG][SCR];
  __shared__ __align__(16) uint16_t ring[NG][kP2Stages][B];
  // |w| maxima of the salient values per tile row (fp64 bit patterns,
  // ordered as unsigned integers), double-buffered by tile parity
  __shared__ unsigned long long s_rmax2[2][kTileRowsMax];
  __shared__ int s_tile[4];
  extern __shared__ __align__(16) double stash_s[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gw = lane / P, t = lane % P;
  const int g = warp * GPW + gw;
  const int M = p.M, K = p.K, n_sal = p.n_sal, R = p.R, rshift = p.rshift;
  const int ipg = p.ipg, ntiles = p.ntiles;
  const int item0 = g * ipg;
  const double c = p.c;
  const double kInv7 = 1.0 / 7.0, kInv127 = 1.0 / 127.0;
  double *const sgrp = scratch[g];

  if (tid == 0) {
    s_tile[0] = (int)atomicAdd(p.tile_ctr, 1u);
    s_tile[1] = (int)atomicAdd(p.tile_ctr, 1u);
  }
  for (int i = tid; i < 2 * kTileRowsMax; i += blockDim.x) s_rmax2[i >> 6][i & 63] = 0ull;
  __syncthreads();
  int cur = s_tile[0], nxt = s_tile[1];

  // source of row-block ii of this group in tile `tile` (nullptr: none)
  auto src_of = [&](int tile, int ii) -> const uint16_t * {
    if (tile >= ntiles) return nullptr;
    const int item = item0 + ii;
    const int kb = item >> rshift;
    const int row = (tile << rshift) + (item - (kb << rshift));
    if (row >= M) return nullptr;
    return p.W + (size_t)row * K + (size_t)kb * B;
  };
  auto issue = [&](const uint16_t *src, int slot) {
    if (src != nullptr) {
      uint16_t *dst = ring[g][slot];
#pragma unroll
      for (int q = t; q < PIECES; q += P) cp_async16(dst + q * 8, src + q * 8);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < kP2Stages - 1; ++s) issue(src_of(cur, s), s);

  // Salient tables, built once per CTA (a CTA's groups meet the same column
  // blocks in every tile): each block's first entry in sal_idx (and n_sal
  // at the end) and each entry's position in the staged row.
  int16_t *tab_pos = reinterpret_cast<int16_t *>(stash_s + (p.stash_smem ? (size_t)R * n_sal : 0));
  int *tab_pref = reinterpret_cast<int *>(tab_pos + ((n_sal + 3) & ~3));
  unsigned long long unsafe = 0;
  bool sal_ready = false;   // the salient set (from the select kernel) is visible
  int pos = 0;    // ring position of the row-block in hand
  int k = 0;      // tiles done by this CTA: parity of the next-tile slots
  while (cur < ntiles) {
    if (tid == 0) s_tile[2 + (k & 1)] = (int)atomicAdd(p.tile_ctr, 1u);   // the tile after nxt
    double *const stash = p.stash_smem ? stash_s : nullptr;
    for (int ii = 0; ii < ipg; ++ii, ++pos) {
      const int item = item0 + ii;
      const int kb = item >> rshift, r = item - (kb << rshift);
      const int row = (cur << rshift) + r;
      const bool valid = row < M;
      // the exact-path mask of this row-block (written by pass 1, which
      // completed before the select kernel released this one; read from L2),
      // loaded first so that its latency overlaps the ring wait and the rotation
      const uint32_t mk = valid ? __ldcg(p.xmask + (size_t)(row >> 4) * (K / B) + kb) : 0u;
      const int ia = ii + kP2Stages - 1;
      issue(ia < ipg ? src_of(cur, ia) : src_of(nxt, ia - ipg), (pos + kP2Stages - 1) % kP2Stages);
      cp_async_wait<kP2Stages - 1>();
      __syncwarp();
      const uint16_t *buf = ring[g][pos % kP2Stages];
      double v[16];
#pragma unroll
      for (int a = 0; a < 16; ++a) v[a] = bf16_bits_to_f64(buf[P * a + t]);
      fwht_group<B>(v, sgrp, t);
      // row-blocks that pass 1 flagged: exact integer sums, rounded once
      if (valid) {
        if (((mk >> (row & 15)) & 1u) && !block_has_nonfinite(buf, B)) {
          exact_pm_sums16(buf, B, t, sgrp);         // free until the staging below
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = sgrp[16 * t + j];
        }
      }
      // v holds the values the codes see: unscaled sums (b = 256) or w = c * sum
      if (!kPow2) {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __dmul_rn(v[j], c);
      }
      double2 *stg = reinterpret_cast<double2 *>(sgrp + 16 * t);
#pragma unroll
      for (int m = 0; m < 8; ++m) stg[m ^ (t & 7)] = make_double2(v[2 * m], v[2 * m + 1]);
      __syncwarp();
      // this block's salient columns: to the stash, then zero in the staged row
      // everything above (tile claims, the W ring, the rotation) is
      // independent of the salient set and overlaps the select kernel.  The
      // salient set is read with plain loads (cached in L1: the rows of a
      // column block reuse it): a read-only-cache load counts as invariant
      // over the kernel and may be hoisted above the wait.
      if (!sal_ready) {
        pdl_wait();
        // every thread of the CTA is here, in its first row-block
        for (int e = tid; e < n_sal; e += blockDim.x)
          tab_pos[e] = (int16_t)stage_pos(p.sal_idx[e] & (B - 1));
        const int nkb = K / B;
        for (int k = tid; k <= nkb; k += blockDim.x)
          tab_pref[k] = k < nkb ? p.sal_prefix[(k * B) >> 5] : n_sal;
        __syncthreads();
        sal_ready = true;
      }
      const int e0 = tab_pref[kb], e1 = tab_pref[kb + 1];
      double lm = 0.0;                    // this thread's share of the row's salient |w| max
      if (valid && e0 < e1) {
        double *dst = stash != nullptr ? stash + (size_t)r * n_sal : p.sv + (size_t)row * n_sal;
        for (int e = e0 + t; e < e1; e += P) {
          const int si = tab_pos[e];
          const double w = sgrp[si];
          dst[e] = w;
          lm = fmax(lm, fabs(w));
          sgrp[si] = 0.0;
        }
      }
#pragma unroll
      for (int o = 1; o < P; o <<= 1) lm = fmax(lm, __shfl_xor_sync(0xffffffffu, lm, o));
      if (t == 0 && lm > 0.0)
        atomicMax(&s_rmax2[k & 1][r], (unsigned long long)__double_as_longlong(lm));
      __syncwarp();
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const double2 d = stg[m ^ (t & 7)];
        v[2 * m] = d.x;
        v[2 * m + 1] = d.y;
      }
      // group absmax over 64 columns = 4 threads
      double amax = 0.0;
#pragma unroll
      for (int j = 0; j < 16; ++j) amax = fmax(amax, fabs(v[j]));
      amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // absmax of w = c * amax (exact for b = 256)
      const uint16_t sbits = bf16_of_quotient(kPow2 ? amax * c : amax, 7.0, kInv7);
      const double s = bf16_bits_to_f64(sbits);
      const double inv = s > 0.0 ? recip_bf16(sbits) : 0.0;
      const double vinv = kPow2 ? inv * c : inv;    // multiplies v
      // RN64 is monotone, so max_j |RN64(v_j vinv)| = RN64(amax vinv); below
      // 7.5 every code is in [-7, 7] and rint is the add of 1.5 * 2^52 (exact
      // round-half-even to an integer whose two's complement is the low word)
      uint32_t lo[16];
      if (__dmul_rn(amax, vinv) < 7.5) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          lo[j] = (uint32_t)__double2loint(__dadd_rn(__dmul_rn(v[j], vinv), 0x1.8p52));
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          lo[j] = (uint32_t)min(7, max(-8, __double2int_rn(__dmul_rn(v[j], vinv))));
      }
      if (valid) {
        const int col0 = kb * B + 16 * t;
        *reinterpret_cast<uint2 *>(p.q4 + (size_t)row * (K / 2) + (col0 >> 1)) =
            make_uint2(pack_nibbles8(lo), pack_nibbles8(lo + 8));
        if ((t & 3) == 0) {
          p.s4[(size_t)row * (K / 64) + (col0 >> 6)] = sbits;
          if (s > 0.0 && (s < 0x1p-17 || s > 8188.0)) ++unsafe;
        }
        if (RESID) {
          float rres[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const double w = kPow2 ? v[j] * c : v[j];
            rres[j] = (float)__dsub_rn(w, (double)(int)lo[j] * s);
          }
          float4 *rdst = reinterpret_cast<float4 *>(p.resid + (size_t)row * K + col0);
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            rdst[j / 4] = make_float4(rres[j], rres[j + 1], rres[j + 2], rres[j + 3]);
        }
      }
      __syncwarp();
    }

    // INT8 tier of the tile's rows: s8 = bf16_rn(max|w| / 127), q8 = clip(rint(w / s8))
    __syncthreads();                      // the tile's stash and row maxima are complete
    const int n8 = n_sal >> 3;
    const double vscale = kPow2 ? c : 1.0;
    unsigned long long *s_rmax = s_rmax2[k & 1];
    for (int ch = tid; ch < (n8 << rshift); ch += blockDim.x) {
      const int r = ch / n8, e = (ch - r * n8) * 8;
      const int row = (cur << rshift) + r;
      if (row >= M) continue;
      const double2 *src = reinterpret_cast<const double2 *>(
          (stash != nullptr ? stash + (size_t)r * n_sal : p.sv + (size_t)row * n_sal) + e);
      const double m = __longlong_as_double((long long)s_rmax[r]) * vscale;
      const uint16_t sb = bf16_of_quotient(m, 127.0, kInv127);
      const double s8v = bf16_bits_to_f64(sb);
      const double vinv = s8v > 0.0 ? recip_bf16(sb) * vscale : 0.0;
      uint32_t pk[2] = {0u, 0u};
      // w vinv is either NaN (a non-finite weight; it codes to -128, as
      // rint's integer conversion gives) or at most 127.5 in magnitude: rint
      // is then the add of 1.5 * 2^52 (exact round-half-even, the integer in
      // the low word)
      auto q8_of = [&](double w) {
        const double x = __dmul_rn(w, vinv);
        const int q = __double2loint(__dadd_rn(x, 0x1.8p52));
        return x != x ? -128 : min(127, max(-128, q));
      };
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const double2 d = src[u];
        const int qa = q8_of(d.x);
        const int qb = q8_of(d.y);
        pk[u >> 1] |= (((uint32_t)qa & 0xFFu) | (((uint32_t)qb & 0xFFu) << 8)) << (16 * (u & 1));
      }
      *reinterpret_cast<uint2 *>(p.q8 + (size_t)row * n_sal + e) = make_uint2(pk[0], pk[1]);
      if (e == 0) {
        p.s8[row] = sb;
        if (s8v > 0.0 && (s8v < 0x1p-17 || s8v > 511.0)) ++unsafe;
      }
    }
    if (n8 == 0)
      for (int r = tid; r < R; r += blockDim.x)
        if ((cur << rshift) + r < M) p.s8[(cur << rshift) + r] = 0;
    __syncthreads();                      // the stash is free for the next tile
    // this buffer serves tile k + 2, whose stash starts after tile k + 1's barriers
    if (tid < R) s_rmax[tid] = 0ull;
    cur = nxt;
    nxt = s_tile[2 + (k & 1)];
    ++k;
  }
  cp_async_wait<0>();
  if (unsafe) atomicAdd(&p.info[1], unsafe);
}

// --------------------------------------------------------------- launch ---
namespace {
constexpr int groups_per_cta(int B) { return (32 / (B / 16)) * 4; }

struct Pass2Plan {
  int R, rshift, ipg, ntiles;
  bool smem;
  size_t smem_bytes;
};
// shared memory of pass 2's salient tables: n_sal positions, nkb + 1 block starts
size_t sal_tab_bytes(int n_sal, int nkb) {
  return (size_t)((n_sal + 3) & ~3) * sizeof(int16_t) + (size_t)(nkb + 1) * sizeof(int);
}
constexpr size_t kSalTabMax = (size_t)kMaxSalient * 2 + (65536 / 128 + 1) * 4;

// Rows per tile: the smallest power of two that splits the tile's R * nkb
// row-blocks evenly over the groups with at least kP2Stages - 1 per group.
Pass2Plan pass2_plan(int M, int K, int B, int n_sal) {
  const int NG = groups_per_cta(B), nkb = K / B;
  int R = 1;
  while ((R * nkb) % NG != 0 || R * nkb / NG < kP2Stages - 1) R *= 2;
  Pass2Plan pl{};
  pl.R = R;
  pl.rshift = 0;
  while ((1 << pl.rshift) < R) ++pl.rshift;
  pl.ipg = R * nkb / NG;
  pl.ntiles = (M + R - 1) / R;
  const size_t bytes = (size_t)R * n_sal * sizeof(double);
  pl.smem = bytes <= (size_t)kStashSmemMax;
  pl.smem_bytes = pl.smem ? bytes : 0;
  pl.smem_bytes += sal_tab_bytes(n_sal, nkb);
  return pl;
}

struct EncodeLayout {
  size_t info, ctr, done, zero_bytes, gpart, score, pref, sv, xmask, total;
};
EncodeLayout encode_layout(int M, int K, int block, int n_sal) {
  const size_t nchunk = (size_t)(M + kSsqChunk - 1) / kSsqChunk;
  const size_t nsg = (nchunk + kSsqGroup - 1) / kSsqGroup;
  const Pass2Plan pl = pass2_plan(M, K, block, n_sal);
  EncodeLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  // counters zeroed at the start of every encode: info[4], tile counter, done[nkb]
  L.info = take(4 * sizeof(unsigned long long) + sizeof(unsigned int) +
                (size_t)(K / block) * sizeof(unsigned int));
  L.ctr = L.info + 4 * sizeof(unsigned long long);
  L.done = L.ctr + sizeof(unsigned int);
  L.zero_bytes = 4 * sizeof(unsigned long long) + sizeof(unsigned int) +
                 (size_t)(K / block) * sizeof(unsigned int);
  L.gpart = take(nsg * (size_t)K * sizeof(double));
  L.score = take((size_t)K * sizeof(double));
  L.pref = take((size_t)((K + 31) / 32) * sizeof(int32_t));
  L.sv = take(pl.smem ? 0 : (size_t)M * n_sal * sizeof(double));
  L.xmask = take(nchunk * (size_t)(K / block) * sizeof(uint16_t));
  L.total = off;
  return L;
}

template <int B, bool RESID>
cudaError_t launch_pass2(const Pass2Params &pp, size_t smem, cudaStream_t st, Launcher &L) {
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, enc_pass2_kernel<B, RESID>,
                                                                128, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const long long grid = std::max(1LL, std::min<long long>(pp.ntiles, (long long)nsm * occ));
  return L.launch("enc_pass2", enc_pass2_kernel<B, RESID>, dim3((unsigned)grid), dim3(128), smem,
                  st, true, pp);
}
}  // namespace

size_t encode_workspace_bytes(int M, int K, int block, int n_sal) {
  return encode_layout(M, K, block, n_sal).total;
}

cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t st, Launcher &L) {
  const int M = a.M, K = a.K, B = a.block;
  const int nchunk = (M + kSsqChunk - 1) / kSsqChunk;
  const EncodeLayout lay = encode_layout(M, K, B, a.n_sal);
  const Pass2Plan pl = pass2_plan(M, K, B, a.n_sal);
  char *ws = static_cast<char *>(a.workspace);
  auto *info = reinterpret_cast<unsigned long long *>(ws + lay.info);
  auto *ctr = reinterpret_cast<unsigned int *>(ws + lay.ctr);
  auto *done = reinterpret_cast<unsigned int *>(ws + lay.done);
  auto *gpart = reinterpret_cast<double *>(ws + lay.gpart);
  auto *score = reinterpret_cast<double *>(ws + lay.score);
  auto *pref = reinterpret_cast<int32_t *>(ws + lay.pref);
  auto *sv = pl.smem ? nullptr : reinterpret_cast<double *>(ws + lay.sv);
  auto *xmask = reinterpret_cast<uint16_t *>(ws + lay.xmask);
  const double c = sqrt(1.0 / (double)B);

  cudaError_t e = cudaMemsetAsync(info, 0, lay.zero_bytes, st);
  if (e != cudaSuccess) return e;
  const int nkb = K / B;
  const int NG = groups_per_cta(B);
  dim3 g1((unsigned)(((nchunk + NG - 1) / NG) * nkb));
  auto p1 = B == 256 ? enc_pass1_kernel<256> : enc_pass1_kernel<128>;
  e = L.launch("enc_pass1", p1, g1, dim3(128), 0, st, false, (const uint16_t *)a.W, M, K, c,
               a.act_scale, gpart, score, done, info, xmask);
  if (e != cudaSuccess) return e;
  const size_t sel_smem = K <= kSelSmemKeys ? (size_t)K * sizeof(unsigned long long) : 0;
  e = L.launch("enc_select", enc_select_kernel, dim3(1), dim3(kSelThreads), sel_smem, st, true,
               (const double *)score, K, a.n_sal, a.sal_idx, pref);
  if (e != cudaSuccess) return e;

  Pass2Params pp{};
  pp.W = (const uint16_t *)a.W;
  pp.M = M; pp.K = K; pp.n_sal = a.n_sal;
  pp.R = pl.R; pp.rshift = pl.rshift; pp.ipg = pl.ipg; pp.ntiles = pl.ntiles;
  pp.stash_smem = pl.smem ? 1 : 0;
  pp.c = c;
  pp.sal_idx = a.sal_idx; pp.sal_prefix = pref;
  pp.q4 = a.q4; pp.s4 = a.s4; pp.q8 = a.q8; pp.s8 = a.s8; pp.resid = a.resid;
  pp.sv = sv; pp.tile_ctr = ctr; pp.info = info; pp.xmask = xmask;
  if (B == 256)
    e = a.resid ? launch_pass2<256, true>(pp, pl.smem_bytes, st, L)
                : launch_pass2<256, false>(pp, pl.smem_bytes, st, L);
  else
    e = a.resid ? launch_pass2<128, true>(pp, pl.smem_bytes, st, L)
                : launch_pass2<128, false>(pp, pl.smem_bytes, st, L);
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
       {(const void *)enc_pass1_kernel<256>, (const void *)enc_pass1_kernel<128>})
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
  for (const void *f :
       {(const void *)enc_pass2_kernel<256, false>, (const void *)enc_pass2_kernel<128, false>,
        (const void *)enc_pass2_kernel<256, true>, (const void *)enc_pass2_kernel<128, true>}) {
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)(kStashSmemMax + kSalTabMax))) != cudaSuccess)
      return e;
  }
  double recip[128];
  for (int m = 0; m < 128; ++m) recip[m] = 1.0 / (double)(128 + m);
  if ((e = cudaMemcpyToSymbol(kRecipMant, recip, sizeof(recip))) != cudaSuccess) return e;
  return cudaFuncSetAttribute(enc_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kSelSmemKeys * (int)sizeof(unsigned long long));
}

}  // namespace dvssq
