// DV-SSQ encoder kernels (Spark-X2.5-4B-Hadamard-GSQ model card, DV-SSQ
// Tiers A and B; MiniCPM5-2B-Hadamard-GSQ model card, Mathematical
// Foundations §1-§2).
//
//   pass 1  W_rot = W . H_K row-block by row-block in fp64 (exact +-1 sums,
//           one scale by 1/sqrt(b)); per-column sum of squares over fixed
//           chunks of 64 rows; exactness check of every row-block.
//   score   chunk partials summed in ascending order, score = a * sqrt(ssq).
//   select  the n_sal largest scores (ties -> lower index) by an MSB-first
//           radix select in one CTA; outputs sorted indices, a column bit
//           mask and per-32-column prefix counts.
//   pass 2  rotation again, INT4 group RTN with BF16 scales, nibble packing,
//           salient values stashed in shared memory for the row's INT8 scale,
//           INT8 codes; optional fp32 residual.
#include "common.cuh"
#include "fwht_group.cuh"
#include "kernels.h"

namespace dvssq {

constexpr int kSsqChunk = 64;     // rows per fixed-order partial (salience)
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
        double w = __dmul_rn(v[j], c);
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
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      double2 d = make_double2(ssq[j], ssq[j + 1]);
      *reinterpret_cast<double2 *>(dst + j) = d;
    }
    if (t == 0 && inexact) atomicAdd(&info[0], inexact);
  }
}

// ----------------------------------------------------------------- score --
__global__ void enc_score_kernel(const double *__restrict__ part, int nchunk, int K,
                                 const float *__restrict__ act_scale, double *__restrict__ score,
                                 unsigned long long *__restrict__ info) {
  int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  double tot = 0.0;
  for (int ch = 0; ch < nchunk; ++ch) tot = __dadd_rn(tot, part[(size_t)ch * K + j]);
  double s = __dmul_rn((double)act_scale[j], __dsqrt_rn(tot));
  if (!isfinite(s)) atomicAdd(&info[2], 1ull);
  score[j] = s;
}

// ---------------------------------------------------------------- select --
// Order-preserving 64-bit key of a non-NaN double (-0 treated as +0).
__device__ __forceinline__ unsigned long long order_key(double d) {
  if (d == 0.0) d = 0.0;
  unsigned long long u = (unsigned long long)__double_as_longlong(d);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

constexpr int kSelThreads = 1024;

__global__ void __launch_bounds__(kSelThreads) enc_select_kernel(
    const double *__restrict__ score, int K, int n_sal, int32_t *__restrict__ sal_idx,
    uint32_t *__restrict__ sal_mask, int32_t *__restrict__ sal_prefix) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ unsigned int s_krem;
  __shared__ int s_scan[kSelThreads];
  __shared__ int s_scan2[kSelThreads];
  const int tid = threadIdx.x;
  const int per = (K + kSelThreads - 1) / kSelThreads;
  const int j0 = min(K, tid * per), j1 = min(K, j0 + per);

  for (int w = tid; w < (K + 31) / 32; w += kSelThreads) sal_mask[w] = 0u;
  if (n_sal == 0) return;

  unsigned long long prefix = 0, pmask = 0;
  unsigned int krem = (unsigned int)n_sal;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int d = tid; d < 256; d += kSelThreads) hist[d] = 0;
    __syncthreads();
    for (int j = j0; j < j1; ++j) {
      unsigned long long k = order_key(score[j]);
      if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned int cum = 0;
      int d = 255;
      for (; d > 0; --d) {
        if (cum + hist[d] >= krem) break;
        cum += hist[d];
      }
      s_krem = krem - cum;
      s_prefix = prefix | ((unsigned long long)d << shift);
    }
    __syncthreads();
    krem = s_krem;
    prefix = s_prefix;
    pmask |= 255ull << shift;
    __syncthreads();
  }
  // prefix = key of the n_sal-th largest score; krem = how many of the keys
  // equal to it are taken (lowest indices first).
  int n_eq = 0;
  for (int j = j0; j < j1; ++j) n_eq += order_key(score[j]) == prefix;
  s_scan[tid] = n_eq;
  __syncthreads();
  for (int off = 1; off < kSelThreads; off <<= 1) {   // inclusive Hillis-Steele scan
    int v = tid >= off ? s_scan[tid - off] : 0;
    __syncthreads();
    s_scan[tid] += v;
    __syncthreads();
  }
  int eq_before = s_scan[tid] - n_eq;
  int n_sel = 0;
  {
    int eqr = eq_before;
    for (int j = j0; j < j1; ++j) {
      unsigned long long k = order_key(score[j]);
      bool sel = k > prefix || (k == prefix && (unsigned)(eqr++) < krem);
      n_sel += sel;
    }
  }
  s_scan2[tid] = n_sel;
  __syncthreads();
  for (int off = 1; off < kSelThreads; off <<= 1) {
    int v = tid >= off ? s_scan2[tid - off] : 0;
    __syncthreads();
    s_scan2[tid] += v;
    __syncthreads();
  }
  int pos = s_scan2[tid] - n_sel;
  int eqr = eq_before;
  for (int j = j0; j < j1; ++j) {
    unsigned long long k = order_key(score[j]);
    bool sel = k > prefix || (k == prefix && (unsigned)(eqr++) < krem);
    if ((j & 31) == 0) sal_prefix[j >> 5] = pos;
    if (sel && pos < n_sal) {
      sal_idx[pos++] = j;
      atomicOr(&sal_mask[j >> 5], 1u << (j & 31));
    }
  }
}

// ---------------------------------------------------------------- pass 2 --
// One group of P threads per row; the group walks the row's K/B blocks.
// Dynamic shared memory: per group a stash of n_sal doubles.
template <int B>
__global__ void __launch_bounds__(128) enc_pass2_kernel(
    const uint16_t *__restrict__ W, int M, int K, int n_sal, int rows_per_cta, double c,
    const uint32_t *__restrict__ sal_mask, const int32_t *__restrict__ sal_prefix,
    uint8_t *__restrict__ q4, uint16_t *__restrict__ s4, int8_t *__restrict__ q8,
    uint16_t *__restrict__ s8, float *__restrict__ resid, unsigned long long *__restrict__ info) {
  constexpr int P = B / 16;
  constexpr int GPW = 32 / P;
  constexpr int SCR = GroupScratch<B>::kElems;
  constexpr int NGMAX = 8;
  __shared__ double scratch[NGMAX][SCR];
  __shared__ __align__(16) uint16_t ring[NGMAX][kStages][B];
  extern __shared__ double stash_all[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = lane / P, t = lane % P;
  const int g = warp * GPW + gw;
  const int row = blockIdx.x * rows_per_cta + g;
  const bool active = (g < rows_per_cta) && (row < M);
  double *stash = stash_all + (size_t)g * n_sal;
  const int nkb = K / B;

  constexpr int PIECES = B * 2 / 16;
  auto issue = [&](int i) {
    if (active && i < nkb) {
      const uint16_t *src = W + (size_t)row * K + (size_t)i * B;
      uint16_t *dst = ring[g][i % kStages];
#pragma unroll
      for (int p = t; p < PIECES; p += P) cp_async16(dst + p * 8, src + p * 8);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) issue(i);

  double amax8 = 0.0;
  unsigned long long unsafe = 0;
  for (int kb = 0; kb < nkb; ++kb) {
    issue(kb + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();
    double v[16];
    const uint16_t *buf = ring[g][kb % kStages];
#pragma unroll
    for (int a = 0; a < 16; ++a) v[a] = bf16_bits_to_f64(buf[P * a + t]);
    fwht_group<B>(v, scratch[g], t);
    const int col0 = kb * B + 16 * t;
    const uint32_t mword = sal_mask[col0 >> 5];
    const int bit0 = col0 & 31;
    const uint32_t m16 = (mword >> bit0) & 0xFFFFu;
    double amax = 0.0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      v[j] = __dmul_rn(v[j], c);
      if (!((m16 >> j) & 1u)) amax = fmax(amax, fabs(v[j]));
    }
    // 64-column group = 4 consecutive threads
    amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const uint16_t sbits = f64_to_bf16_rn(__ddiv_rn(amax, 7.0));
    const double s = bf16_bits_to_f64(sbits);
    const double inv = s > 0.0 ? __ddiv_rn(1.0, s) : 0.0;
    uint32_t word[2] = {0u, 0u};
    float rres[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      int q = 0;
      if (!((m16 >> j) & 1u)) {
        q = __double2int_rn(__dmul_rn(v[j], inv));
        q = min(7, max(-8, q));
        rres[j] = (float)__dsub_rn(v[j], (double)q * s);
      } else {
        rres[j] = 0.0f;
        const int e = sal_prefix[col0 >> 5] + __popc(mword & ((1u << (bit0 + j)) - 1u));
        if (active && e < n_sal) stash[e] = v[j];
        amax8 = fmax(amax8, fabs(v[j]));
      }
      word[j >> 3] |= ((uint32_t)q & 0xFu) << (4 * (j & 7));
    }
    if (active) {
      *reinterpret_cast<uint2 *>(q4 + (size_t)row * (K / 2) + (col0 >> 1)) =
          make_uint2(word[0], word[1]);
      if ((t & 3) == 0) {
        s4[(size_t)row * (K / 64) + (col0 >> 6)] = sbits;
        if (s > 0.0 && (s < 0x1p-17 || s > 8188.0)) ++unsafe;
      }
      if (resid != nullptr) {
        float4 *dst = reinterpret_cast<float4 *>(resid + (size_t)row * K + col0);
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          dst[j / 4] = make_float4(rres[j], rres[j + 1], rres[j + 2], rres[j + 3]);
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  // INT8 tier: one scale per row from the row's salient maximum
#pragma unroll
  for (int o = 1; o < P; o <<= 1) amax8 = fmax(amax8, __shfl_xor_sync(0xffffffffu, amax8, o));
  __syncwarp();
  const uint16_t s8bits = f64_to_bf16_rn(__ddiv_rn(amax8, 127.0));
  const double sv8 = bf16_bits_to_f64(s8bits);
  const double inv8 = sv8 > 0.0 ? __ddiv_rn(1.0, sv8) : 0.0;
  if (active) {
    for (int e0 = 4 * t; e0 < n_sal; e0 += 4 * P) {
      uint32_t pk = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        int q = __double2int_rn(__dmul_rn(stash[e0 + u], inv8));
        q = min(127, max(-128, q));
        pk |= ((uint32_t)q & 0xFFu) << (8 * u);
      }
      *reinterpret_cast<uint32_t *>(q8 + (size_t)row * n_sal + e0) = pk;
    }
    if (t == 0) {
      s8[row] = s8bits;
      if (sv8 > 0.0 && (sv8 < 0x1p-17 || sv8 > 511.0)) ++unsafe;
    }
  }
  if (active && unsafe) atomicAdd(&info[1], unsafe);
}

// --------------------------------------------------------------- launch ---
size_t encode_workspace_bytes(int M, int K) {
  const size_t nchunk = (size_t)(M + kSsqChunk - 1) / kSsqChunk;
  size_t off = 0;
  auto take = [&](size_t bytes) { off += (bytes + 255) & ~(size_t)255; };
  take(4 * sizeof(unsigned long long));        // info counters
  take(nchunk * (size_t)K * sizeof(double));   // chunk partials
  take((size_t)K * sizeof(double));            // scores
  take((size_t)((K + 31) / 32) * sizeof(uint32_t));   // salient mask
  take((size_t)((K + 31) / 32) * sizeof(int32_t));    // per-word prefix
  return off;
}

cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t st, Launcher &L) {
  const int M = a.M, K = a.K, B = a.block;
  const int nchunk = (M + kSsqChunk - 1) / kSsqChunk;
  char *ws = static_cast<char *>(a.workspace);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char *p = ws + off;
    off += (bytes + 255) & ~(size_t)255;
    return p;
  };
  auto *info = reinterpret_cast<unsigned long long *>(take(4 * sizeof(unsigned long long)));
  auto *part = reinterpret_cast<double *>(take((size_t)nchunk * K * sizeof(double)));
  auto *score = reinterpret_cast<double *>(take((size_t)K * sizeof(double)));
  auto *mask = reinterpret_cast<uint32_t *>(take((size_t)((K + 31) / 32) * sizeof(uint32_t)));
  auto *pref = reinterpret_cast<int32_t *>(take((size_t)((K + 31) / 32) * sizeof(int32_t)));
  const double c = sqrt(1.0 / (double)B);

  cudaError_t e = cudaMemsetAsync(info, 0, 4 * sizeof(unsigned long long), st);
  if (e != cudaSuccess) return e;
  const int nkb = K / B;
  const int P = B / 16, NG = (32 / P) * 4;
  const long long pairs = (long long)nchunk * nkb;
  dim3 g1((unsigned)((pairs + NG - 1) / NG));
  if (B == 256)
    e = L.launch("enc_pass1", enc_pass1_kernel<256>, g1, dim3(128), 0, st, false,
                 (const uint16_t *)a.W, M, K, c, part, info);
  else
    e = L.launch("enc_pass1", enc_pass1_kernel<128>, g1, dim3(128), 0, st, false,
                 (const uint16_t *)a.W, M, K, c, part, info);
  if (e != cudaSuccess) return e;
  e = L.launch("enc_score", enc_score_kernel, dim3((K + 255) / 256), dim3(256), 0, st, false,
               (const double *)part, nchunk, K, a.act_scale, score, info);
  if (e != cudaSuccess) return e;
  e = L.launch("enc_select", enc_select_kernel, dim3(1), dim3(kSelThreads), 0, st, false,
               (const double *)score, K, a.n_sal, a.sal_idx, mask, pref);
  if (e != cudaSuccess) return e;
  const int rows_per_cta = pass2_rows_per_cta(B, a.n_sal);
  const int threads = ((rows_per_cta * P + 31) / 32) * 32;
  const size_t dsmem = (size_t)rows_per_cta * a.n_sal * sizeof(double);
  dim3 g2((unsigned)((M + rows_per_cta - 1) / rows_per_cta));
  if (B == 256) {
    e = L.launch("enc_pass2", enc_pass2_kernel<256>, g2, dim3(threads), dsmem, st, false,
                 (const uint16_t *)a.W, M, K, a.n_sal, rows_per_cta, c, (const uint32_t *)mask,
                 (const int32_t *)pref, a.q4, a.s4, a.q8, a.s8, a.resid, info);
  } else {
    e = L.launch("enc_pass2", enc_pass2_kernel<128>, g2, dim3(threads), dsmem, st, false,
                 (const uint16_t *)a.W, M, K, a.n_sal, rows_per_cta, c, (const uint32_t *)mask,
                 (const int32_t *)pref, a.q4, a.s4, a.q8, a.s8, a.resid, info);
  }
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

int pass2_rows_per_cta(int block, int n_sal) {
  // Rows (one per thread group) whose salient stash fits 96 KB of shared
  // memory, so that two CTAs share an SM; one row for the largest sets.
  (void)block;
  for (int rows = 8; rows > 1; rows >>= 1)
    if ((size_t)rows * n_sal * sizeof(double) <= 96 * 1024) return rows;
  return 1;
}

cudaError_t prepare_encode_kernels() {
  // pass 2 may use up to 8 rows x n_sal doubles of dynamic shared memory
  cudaError_t e = cudaFuncSetAttribute(enc_pass2_kernel<256>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(enc_pass2_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              160 * 1024);
}

}  // namespace dvssq
