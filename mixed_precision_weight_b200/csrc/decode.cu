// Decode-shaped forward (T <= 16 tokens) of the DV-SSQ layer: the runtime
// equation of the MiniCPM5-2B-Hadamard-GSQ card (§2, Y = X What^T + (X B^T)
// A^T) with the Spark card's INT8 salient tier, on the packed form.
//
// Two launches, chained by programmatic dependent launch:
//   dec_prologue  one CTA per Hadamard block: xr = H_b x in fp32 (16-thread
//                 Kronecker FWHT), written as FP16 in the GEMV's k-order; the
//                 salient entries xs = xr[sal_idx]; the block's partial of
//                 t = V xr; zeroes the split-K arrival counters.
//   dec_main      CTA tile = 64 rows x (1024 * NR) columns.  TMA brings the
//                 CTA's whole q8 slice (64B swizzle) and q4 tile (128B
//                 swizzle) into shared memory at once, before the kernel
//                 waits on the prologue, so the weight stream overlaps it.
//                 Each warp owns 128-column slices of all 64 rows.  The
//                 salient tier runs first: exact FP16 INT8 codes x xs on
//                 mma.sync, scaled by s8 in FP32.  Then per 64-column group:
//                 nibbles -> exact FP16 codes in registers -> mma.sync
//                 m16n8k16 with FP32 accumulation -> acc += s4 * group sum.
//                 Warps reduce in shared memory and the CTA adds U (its own
//                 slice of t), so split-K partials sum to the whole layer.
//                 One k-split writes y directly; otherwise the last CTA of a
//                 row block sums the partials in k order (deterministic).
#include "common.cuh"
#include "fwht_group.cuh"
#include "kernels.h"

#include <stdlib.h>

namespace dvssq {

constexpr int kDecBM = 64;
constexpr int kDecRound = 1024;          // columns of one round (8 warps x 128)
constexpr int kDecThreads = 256;
constexpr int kDecQ4Box = 64 * 128;      // bytes of one q4 box (64 rows x 256 cols)
constexpr int kDecQ8Box = 64 * 64;       // bytes of one q8 box (64 rows x 64 entries)
constexpr int kDecMaxNR = 4;

struct DecodeParams {
  int M, K, T, n_sal, rank, block, nkb, NR, BK, KT, RB, SE, nq8box;
  int s4_tma, u_tma;          // 1 when the scale / U tables come by TMA
  float c;
  const uint16_t *s4;
  const int32_t *sal_idx;
  const uint16_t *s8;
  const uint16_t *U;
  const uint16_t *V;
  const uint16_t *x;
  const uint16_t *bias;
  void *y;
  int y_bf16;
  __half *xr16;
  __half *xs16;
  float *tp;
  float *part;
  unsigned int *counters;
};

// Position i of each 16-column segment of xr16 holds column perm16(i): the
// order in which nibble pairs come out of the dequantiser (see dequant_q4),
// i.e. {0,4,1,5, 2,6,3,7, 8,12,9,13, 10,14,11,15}.
__host__ __device__ constexpr int perm16(int i) {
  return (i & 8) | ((i & 1) << 2) | ((i >> 1) & 3);
}

// ------------------------------------------------------------- prologue ---
// Dynamic shared memory: V block [rank][B + 8] FP16 (converted from BF16).
template <int B>
__global__ void __launch_bounds__(B) dec_prologue_kernel(DecodeParams p) {
  pdl_launch_dependents();
  constexpr int P = B / 16;
  __shared__ float scratch[16][GroupScratch<B>::kElems];
  __shared__ float xr[16][B + 1];
  __shared__ __align__(16) __half xh[16][B + 8];
  __shared__ int s_cnt[2];
  extern __shared__ __align__(16) uint8_t vs_raw[];
  __half(*vh)[B + 8] = reinterpret_cast<__half(*)[B + 8]>(vs_raw);

  const int kb = blockIdx.x, tid = threadIdx.x;
  const int tok = tid / P, t = tid % P;
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, tig = lane & 3;
  const bool live = tok < p.T;
  if (tid < 2) s_cnt[tid] = 0;

  // issue every global load first: x, V, sal_idx
  uint16_t xin[16];
#pragma unroll
  for (int a = 0; a < 16; ++a)
    xin[a] = live ? p.x[(size_t)tok * p.K + (size_t)kb * B + P * a + t] : (uint16_t)0;
  constexpr int VPT = 64 * B / 8 / B;            // uint4 per thread for rank <= 64
  uint4 vreg[VPT];
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int i = tid + u * B;
    const int rr = i / (B / 8), cc = i % (B / 8);
    vreg[u] = rr < p.rank ? *reinterpret_cast<const uint4 *>(p.V + (size_t)rr * p.K +
                                                             (size_t)kb * B + cc * 8)
                          : make_uint4(0, 0, 0, 0);
  }
  int lo = 0, hi = 0;
  for (int e = tid; e < p.n_sal; e += B) {
    const int s = p.sal_idx[e];
    lo += s < kb * B;
    hi += s < (kb + 1) * B;
  }
  if (kb == 0)
    for (int i = tid; i < p.RB; i += B) p.counters[i] = 0u;

  float v[16];
#pragma unroll
  for (int a = 0; a < 16; ++a) v[a] = bf16_bits_to_f32(xin[a]);
  // whole warps whose tokens are all beyond T skip the transform
  const bool warp_live = (tid & ~31) / P < p.T;
  if (warp_live) {
    fwht_group<B>(v, scratch[tok], t);
    uint32_t hn[8];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      v[j] *= p.c;
      xr[tok][16 * t + j] = v[j];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      hn[i] = pack_half2(__float2half_rn(v[2 * i]), __float2half_rn(v[2 * i + 1]));
    *reinterpret_cast<uint4 *>(&xh[tok][16 * t]) = make_uint4(hn[0], hn[1], hn[2], hn[3]);
    *reinterpret_cast<uint4 *>(&xh[tok][16 * t + 8]) = make_uint4(hn[4], hn[5], hn[6], hn[7]);
    if (live) {
      uint32_t h[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        h[i] = pack_half2(__float2half_rn(v[perm16(2 * i)]), __float2half_rn(v[perm16(2 * i + 1)]));
      uint4 *dst = reinterpret_cast<uint4 *>(p.xr16 + (size_t)tok * p.K + (size_t)kb * B + 16 * t);
      dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
      dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
    }
  } else {
    *reinterpret_cast<uint4 *>(&xh[tok][16 * t]) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(&xh[tok][16 * t + 8]) = make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int i = tid + u * B;
    const int rr = i / (B / 8), cc = i % (B / 8);
    if (rr < p.rank) {
      const uint32_t w[4] = {vreg[u].x, vreg[u].y, vreg[u].z, vreg[u].w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = pack_half2(__float2half_rn(bf16_bits_to_f32(w[q] & 0xFFFFu)),
                          __float2half_rn(bf16_bits_to_f32(w[q] >> 16)));
      *reinterpret_cast<uint4 *>(&vh[rr][cc * 8]) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
  if (lo) atomicAdd(&s_cnt[0], lo);
  if (hi) atomicAdd(&s_cnt[1], hi);
  // this block's partial of t = V xr (tokens x ranks) on mma.sync, one n-tile
  // of 8 ranks per warp
  for (int nt = warp; nt < (p.rank + 7) / 8; nt += B / 32) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int n = 8 * nt + g;
#pragma unroll 4
    for (int k0 = 0; k0 < B; k0 += 16) {
      uint32_t a[4];
      a[0] = *reinterpret_cast<const uint32_t *>(&xh[g][k0 + 2 * tig]);
      a[1] = *reinterpret_cast<const uint32_t *>(&xh[g + 8][k0 + 2 * tig]);
      a[2] = *reinterpret_cast<const uint32_t *>(&xh[g][k0 + 2 * tig + 8]);
      a[3] = *reinterpret_cast<const uint32_t *>(&xh[g + 8][k0 + 2 * tig + 8]);
      const uint32_t b0 = n < p.rank ? *reinterpret_cast<const uint32_t *>(&vh[n][k0 + 2 * tig]) : 0u;
      const uint32_t b1 = n < p.rank ? *reinterpret_cast<const uint32_t *>(&vh[n][k0 + 2 * tig + 8]) : 0u;
      mma_16816(acc, a, b0, b1, acc);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = g + 8 * (i >> 1), rr = 8 * nt + 2 * tig + (i & 1);
      if (q < p.T && rr < p.rank) p.tp[((size_t)kb * p.rank + rr) * p.T + q] = acc[i];
    }
  }
  __syncthreads();
  // salient entries whose rotated column falls in this block
  const int e_lo = s_cnt[0], e_hi = s_cnt[1];
  for (int e = e_lo + tid; e < e_hi; e += B) {
    const int col = p.sal_idx[e] - kb * B;
    if (col < 0 || col >= B) continue;   // sal_idx must be sorted; ignore otherwise
    for (int q = 0; q < p.T; ++q)
      p.xs16[(size_t)q * p.n_sal + e] = __float2half_rn(xr[q][col]);
  }
}

// ----------------------------------------------------------------- main ---
// 8 nibbles of a 32-bit word (biased by XOR 8, i.e. u = q + 8) -> four FP16
// pairs holding the exact codes q: (n0,n4), (n1,n5), (n2,n6), (n3,n7).
__device__ __forceinline__ void dequant_q4(uint32_t w, uint32_t out[4]) {
  const uint32_t u = w ^ 0x88888888u;
  const uint32_t magic = 0x64006400u;               // FP16 1024 in both halves
  const __half2 sub_lo = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));  // 1032
  const __half2 mul_hi = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));  // 1/16
  const __half2 sub_hi = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));  // -72
  uint32_t l0 = (u & 0x000F000Fu) | magic;
  uint32_t h0 = (u & 0x00F000F0u) | magic;
  uint32_t l1 = ((u >> 8) & 0x000F000Fu) | magic;
  uint32_t h1 = ((u >> 8) & 0x00F000F0u) | magic;
  __half2 r0 = __hsub2(*reinterpret_cast<__half2 *>(&l0), sub_lo);
  __half2 r1 = __hfma2(*reinterpret_cast<__half2 *>(&h0), mul_hi, sub_hi);
  __half2 r2 = __hsub2(*reinterpret_cast<__half2 *>(&l1), sub_lo);
  __half2 r3 = __hfma2(*reinterpret_cast<__half2 *>(&h1), mul_hi, sub_hi);
  out[0] = *reinterpret_cast<uint32_t *>(&r0);
  out[1] = *reinterpret_cast<uint32_t *>(&r1);
  out[2] = *reinterpret_cast<uint32_t *>(&r2);
  out[3] = *reinterpret_cast<uint32_t *>(&r3);
}

// 4 int8 codes -> two FP16 pairs (e0,e1), (e2,e3), exact.
__device__ __forceinline__ void dequant_q8(uint32_t w, uint32_t &p01, uint32_t &p23) {
  const uint32_t u = w ^ 0x80808080u;               // q + 128 in [0, 255]
  uint32_t a = __byte_perm(u, 0x64646464u, 0x4140);
  uint32_t b = __byte_perm(u, 0x64646464u, 0x4342);
  const __half2 sub = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));  // 1152
  __half2 ra = __hsub2(*reinterpret_cast<__half2 *>(&a), sub);
  __half2 rb = __hsub2(*reinterpret_cast<__half2 *>(&b), sub);
  p01 = *reinterpret_cast<uint32_t *>(&ra);
  p23 = *reinterpret_cast<uint32_t *>(&rb);
}

// B fragments (activations, FP16, GEMV k-order) of one 128-column slice for
// n-tiles 0..NT-1: [group][ntile][8 registers].
template <int NT>
__device__ __forceinline__ void load_x_frags(const DecodeParams &p, int kw, int g, int tig,
                                             uint32_t bq[2][NT][8]) {
#pragma unroll
  for (int gi = 0; gi < 2; ++gi)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tok = g + 8 * nt;
      const int kc = kw + 64 * gi + 16 * tig;
      if (tok < p.T && kc < p.K) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.xr16 + (size_t)tok * p.K + kc);
        const uint4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
        bq[gi][nt][0] = x0.x; bq[gi][nt][1] = x0.y; bq[gi][nt][2] = x0.z; bq[gi][nt][3] = x0.w;
        bq[gi][nt][4] = x1.x; bq[gi][nt][5] = x1.y; bq[gi][nt][6] = x1.z; bq[gi][nt][7] = x1.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) bq[gi][nt][i] = 0u;
      }
    }
}

// One 128-column slice (two 64-column groups) of the INT4 tier for the four
// 16-row tiles: acc += s4 * (codes x activations).
template <int NT>
__device__ __forceinline__ void int4_slice(const uint8_t *bx, const uint16_t *ss4, int GPC,
                                           int sgrp0, int half, int g, int tig,
                                           const uint32_t bq[2][NT][8], float acc[4][NT][4]) {
  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int gi = 0; gi < 2; ++gi) {
    const int chunk = 4 * half + 2 * gi + (tig >> 1);
    const int sgrp = sgrp0 + gi;
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
      const int rlo = 16 * rt + g;
      const uint32_t off = (uint32_t)(((chunk ^ (rlo & 7)) << 4) + 8 * (tig & 1));
      const uint2 wl = *reinterpret_cast<const uint2 *>(bx + rlo * 128 + off);
      const uint2 wh = *reinterpret_cast<const uint2 *>(bx + (rlo + 8) * 128 + off);
      uint32_t fl[8], fh[8];
      dequant_q4(wl.x, fl);
      dequant_q4(wl.y, fl + 4);
      dequant_q4(wh.x, fh);
      dequant_q4(wh.y, fh + 4);
      const float slo = bf16_bits_to_f32(ss4[rlo * GPC + sgrp]);
      const float shi = bf16_bits_to_f32(ss4[(rlo + 8) * GPC + sgrp]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float d[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t a[4] = {fl[2 * s], fh[2 * s], fl[2 * s + 1], fh[2 * s + 1]};
          mma_16816(d, a, bq[gi][nt][2 * s], bq[gi][nt][2 * s + 1], s == 0 ? zero4 : d);
        }
        acc[rt][nt][0] = fmaf(slo, d[0], acc[rt][nt][0]);
        acc[rt][nt][1] = fmaf(slo, d[1], acc[rt][nt][1]);
        acc[rt][nt][2] = fmaf(shi, d[2], acc[rt][nt][2]);
        acc[rt][nt][3] = fmaf(shi, d[3], acc[rt][nt][3]);
      }
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(kDecThreads, NT == 1 ? 3 : 2) dec_main_kernel(
    const __grid_constant__ CUtensorMap mq4, const __grid_constant__ CUtensorMap mq8,
    const __grid_constant__ CUtensorMap ms4, const __grid_constant__ CUtensorMap mu,
    DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int nbox = 4 * p.NR;
  const int GPC = 16 * p.NR;
  uint8_t *sq4 = base;                                                  // nbox boxes
  uint8_t *sq8 = base + nbox * kDecQ4Box;                               // nq8box boxes
  uint16_t *ss4 = reinterpret_cast<uint16_t *>(sq8 + p.nq8box * kDecQ8Box);   // [64][GPC]
  uint16_t *su = ss4 + kDecBM * GPC;                                    // [64][rank]
  float *tps = reinterpret_cast<float *>(su + kDecBM * 64);             // [rank][T]
  float *s8s = tps + 64 * 16;                                           // [64]
  uint64_t *bars = reinterpret_cast<uint64_t *>(s8s + kDecBM);          // nbox + 2
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int rb = blockIdx.x, kt = blockIdx.y;
  const int m0 = rb * kDecBM, k0 = kt * p.BK, e0 = kt * p.SE;
  const int nsal_cta = max(0, min(p.SE, p.n_sal - e0));
  const bool s4_tma = p.s4_tma != 0, u_tma = p.u_tma != 0 && p.rank > 0;

  if (tid == 0) {
    for (int i = 0; i < nbox + 2; ++i) mbar_init(&bars[i], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    // small per-CTA tables first, then the salient slice, then the INT4 tile
    uint32_t small = (s4_tma ? kDecBM * GPC * 2 : 0) + (u_tma ? kDecBM * p.rank * 2 : 0);
    if (small) {
      mbar_arrive_expect_tx(&bars[nbox + 1], small);
      if (s4_tma) tma_load_2d(ss4, &ms4, k0 / 64, m0, &bars[nbox + 1]);
      if (u_tma) tma_load_2d(su, &mu, 0, m0, &bars[nbox + 1]);
    }
    if (nsal_cta > 0) {
      const int nb = (nsal_cta + 63) / 64;
      mbar_arrive_expect_tx(&bars[nbox], nb * kDecQ8Box);
      for (int i = 0; i < nb; ++i)
        tma_load_2d(sq8 + i * kDecQ8Box, &mq8, e0 + 64 * i, m0, &bars[nbox]);
    }
    for (int box = 0; box < nbox; ++box) {
      if (k0 + 256 * box < p.K) {
        mbar_arrive_expect_tx(&bars[box], kDecQ4Box);
        tma_load_2d(sq4 + box * kDecQ4Box, &mq4, (k0 + 256 * box) / 2, m0, &bars[box]);
      }
    }
  }
  // tables the tensor maps cannot carry (unaligned row strides), and s8
  const int KG = p.K / 64;
  for (int r = warp; r < kDecBM; r += 8) {
    const int row = m0 + r;
    if (!s4_tma)
      for (int gi = lane; gi < GPC; gi += 32) {
        const int gcol = k0 / 64 + gi;
        ss4[r * GPC + gi] = (row < p.M && gcol < KG) ? p.s4[(size_t)row * KG + gcol] : (uint16_t)0;
      }
    if (!u_tma)
      for (int rr = lane; rr < p.rank; rr += 32)
        su[r * p.rank + rr] = row < p.M ? p.U[(size_t)row * p.rank + rr] : (uint16_t)0;
    if (lane == 0) s8s[r] = (row < p.M && p.n_sal > 0) ? bf16_bits_to_f32(p.s8[row]) : 0.0f;
  }

  pdl_wait();   // xr16, xs16, tp and the counters come from the prologue

  // every remaining global load of the warp, issued together
  const int kw0 = k0 + 128 * warp;
  uint32_t bq[2][NT][8];
  load_x_frags<NT>(p, kw0, g, tig, bq);
  const int nsteps = nsal_cta / 16;
  uint32_t sb01[2][NT], sb23[2][NT];     // up to two salient steps per warp
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int st = warp + 8 * j;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tok = g + 8 * nt;
      if (st < nsteps && tok < p.T) {
        const uint2 xv = __ldcg(reinterpret_cast<const uint2 *>(
            p.xs16 + (size_t)tok * p.n_sal + e0 + 16 * st + 4 * tig));
        sb01[j][nt] = xv.x;
        sb23[j][nt] = xv.y;
      } else {
        sb01[j][nt] = 0u;
        sb23[j][nt] = 0u;
      }
    }
  }
  {
    // the CTA's slice of t: sum of the prologue partials of its Hadamard blocks
    const int kb0 = k0 / p.block, kb1 = min(p.nkb, (k0 + p.BK) / p.block);
    const int nkbc = kb1 - kb0;
    for (int i = tid; i < p.rank * p.T; i += kDecThreads) {
      float pv[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        pv[u] = u < nkbc ? __ldcg(&p.tp[(size_t)(kb0 + u) * p.rank * p.T + i]) : 0.0f;
      float sum = 0.0f;
#pragma unroll
      for (int u = 0; u < 16; ++u) sum += pv[u];
      for (int u = 16; u < nkbc; ++u) sum += __ldcg(&p.tp[(size_t)(kb0 + u) * p.rank * p.T + i]);
      tps[i] = sum;
    }
  }
  __syncthreads();   // s8s, fallback tables, tps complete

  float acc[4][NT][4];
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[rt][nt][i] = 0.0f;

  // ---- salient INT8 tier first, into acc, then scaled by s8 ----
  if (warp < nsteps && mbar_wait(&bars[nbox], 0)) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int st = warp + 8 * j;
      if (st >= nsteps) break;
      const uint8_t *bx = sq8 + (st >> 2) * kDecQ8Box;
      const int chunk = st & 3;
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        const int rlo = 16 * rt + g;
        const uint32_t off = (uint32_t)(((chunk ^ ((rlo >> 1) & 3)) << 4) + 4 * tig);
        const uint32_t wl = *reinterpret_cast<const uint32_t *>(bx + rlo * 64 + off);
        const uint32_t wh = *reinterpret_cast<const uint32_t *>(bx + (rlo + 8) * 64 + off);
        uint32_t l01, l23, h01, h23;
        dequant_q8(wl, l01, l23);
        dequant_q8(wh, h01, h23);
        const uint32_t a[4] = {l01, h01, l23, h23};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(acc[rt][nt], a, sb01[j][nt], sb23[j][nt], acc[rt][nt]);
      }
    }
    for (int st = warp + 16; st < nsteps; st += 8) {     // rare: more than two steps
      const uint8_t *bx = sq8 + (st >> 2) * kDecQ8Box;
      const int chunk = st & 3;
      uint32_t b01[NT], b23[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = g + 8 * nt;
        b01[nt] = b23[nt] = 0u;
        if (tok < p.T) {
          const uint2 xv = __ldcg(reinterpret_cast<const uint2 *>(
              p.xs16 + (size_t)tok * p.n_sal + e0 + 16 * st + 4 * tig));
          b01[nt] = xv.x;
          b23[nt] = xv.y;
        }
      }
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        const int rlo = 16 * rt + g;
        const uint32_t off = (uint32_t)(((chunk ^ ((rlo >> 1) & 3)) << 4) + 4 * tig);
        const uint32_t wl = *reinterpret_cast<const uint32_t *>(bx + rlo * 64 + off);
        const uint32_t wh = *reinterpret_cast<const uint32_t *>(bx + (rlo + 8) * 64 + off);
        uint32_t l01, l23, h01, h23;
        dequant_q8(wl, l01, l23);
        dequant_q8(wh, h01, h23);
        const uint32_t a[4] = {l01, h01, l23, h23};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(acc[rt][nt], a, b01[nt], b23[nt], acc[rt][nt]);
      }
    }
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
      const float s8lo = s8s[16 * rt + g], s8hi = s8s[16 * rt + g + 8];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[rt][nt][0] *= s8lo;
        acc[rt][nt][1] *= s8lo;
        acc[rt][nt][2] *= s8hi;
        acc[rt][nt][3] *= s8hi;
      }
    }
  }

  // ---- INT4 tier, one round of 1024 columns at a time ----
  const bool small_ok = !(s4_tma || u_tma) || mbar_wait(&bars[nbox + 1], 0);
  for (int round = 0; round < p.NR && small_ok; ++round) {
    const int kw = kw0 + kDecRound * round;
    if (kw >= p.K) break;
    if (round > 0) load_x_frags<NT>(p, kw, g, tig, bq);
    const int box = 4 * round + (warp >> 1);
    if (!mbar_wait(&bars[box], 0)) break;
    int4_slice<NT>(sq4 + box * kDecQ4Box, ss4, GPC, 16 * round + 2 * warp, warp & 1, g, tig, bq,
                   acc);
  }

  // ---- reduce the 8 warps' k slices in shared memory (reusing the q4 boxes) ----
  __syncthreads();
  float *red = reinterpret_cast<float *>(base);      // [8][64][16]
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int rlo = 16 * rt + g, tok = 2 * tig + 8 * nt;
      red[(warp * 64 + rlo) * 16 + tok] = acc[rt][nt][0];
      red[(warp * 64 + rlo) * 16 + tok + 1] = acc[rt][nt][1];
      red[(warp * 64 + rlo + 8) * 16 + tok] = acc[rt][nt][2];
      red[(warp * 64 + rlo + 8) * 16 + tok + 1] = acc[rt][nt][3];
    }
  __syncthreads();
  for (int i = tid; i < kDecBM * p.T; i += kDecThreads) {
    const int tok = i >> 6, r = i & 63, m = m0 + r;
    if (m >= p.M) continue;
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[(w * 64 + r) * 16 + tok];
    for (int rr = 0; rr < p.rank; ++rr)
      v = fmaf(bf16_bits_to_f32(su[r * p.rank + rr]), tps[rr * p.T + tok], v);
    if (p.KT == 1) {
      if (p.bias) v += bf16_bits_to_f32(p.bias[m]);
      if (p.y_bf16)
        reinterpret_cast<uint16_t *>(p.y)[(size_t)tok * p.M + m] = f32_to_bf16_rn_bits(v);
      else
        reinterpret_cast<float *>(p.y)[(size_t)tok * p.M + m] = v;
    } else {
      p.part[((size_t)kt * p.T + tok) * p.M + m] = v;
    }
  }
  if (p.KT == 1) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.counters[rb], 1u) == (unsigned)(p.KT - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // last CTA of this row block: sum the partials in k order
  for (int i = tid; i < kDecBM * p.T; i += kDecThreads) {
    const int tok = i >> 6, r = i & 63, m = m0 + r;
    if (m >= p.M) continue;
    float v = 0.0f;
    int k = 0;
    for (; k + 8 <= p.KT; k += 8) {
      float pv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) pv[u] = __ldcg(&p.part[((size_t)(k + u) * p.T + tok) * p.M + m]);
#pragma unroll
      for (int u = 0; u < 8; ++u) v += pv[u];
    }
    for (; k < p.KT; ++k) v += __ldcg(&p.part[((size_t)k * p.T + tok) * p.M + m]);
    if (p.bias) v += bf16_bits_to_f32(p.bias[m]);
    if (p.y_bf16)
      reinterpret_cast<uint16_t *>(p.y)[(size_t)tok * p.M + m] = f32_to_bf16_rn_bits(v);
    else
      reinterpret_cast<float *>(p.y)[(size_t)tok * p.M + m] = v;
  }
}

// ---------------------------------------------------------------- host ---
namespace {

struct DecTile {
  int NR, BK, KT, RB, SE, nq8box;
};

// Columns per CTA: one round (1024) by default; two rounds when the grid
// would not fit the resident CTA slots.  DVSSQ_DECODE_ROUNDS overrides it
// (tuning only).
DecTile dec_tile(int M, int K, int n_sal, int T) {
  DecTile d;
  const int RB = (M + kDecBM - 1) / kDecBM;
  // two rounds when the grid would overfill the resident CTA slots, and for
  // T <= 8, where longer k-slices amortise the per-CTA work
  int NR = 1;
  const int slots = 148 * (T <= 8 ? 3 : 2);
  if (K > kDecRound &&
      ((long long)RB * ((K + kDecRound - 1) / kDecRound) > slots || T <= 8))
    NR = 2;
  if (const char *env = getenv("DVSSQ_DECODE_ROUNDS")) {
    const int v = atoi(env);
    if (v >= 1 && v <= kDecMaxNR) NR = v;
  }
  d.NR = NR;
  d.BK = kDecRound * NR;
  d.KT = (K + d.BK - 1) / d.BK;
  d.RB = RB;
  const int boxes = (n_sal + 63) / 64;
  d.SE = n_sal > 0 ? 64 * ((boxes + d.KT - 1) / d.KT) : 0;
  d.nq8box = d.SE / 64;
  return d;
}

size_t dec_smem_bytes(const DecTile &d) {
  return 1024 + (size_t)4 * d.NR * kDecQ4Box + (size_t)d.nq8box * kDecQ8Box +
         (size_t)kDecBM * 16 * d.NR * 2 + (size_t)kDecBM * 64 * 2 + 64 * 16 * 4 + kDecBM * 4 +
         (size_t)(4 * d.NR + 2) * 8;
}

}  // namespace

size_t decode_workspace_bytes(int M, int K, int block, int n_sal, int rank, int T) {
  const DecTile d = dec_tile(M, K, n_sal, T);
  size_t off = 0;
  auto take = [&](size_t b) { off += (b + 255) & ~(size_t)255; };
  take((size_t)T * K * 2);                       // xr16
  take((size_t)T * n_sal * 2 + 16);              // xs16
  take((size_t)(K / block) * rank * T * 4);      // tp
  take((size_t)d.KT * T * M * 4);                // split-K partials
  take((size_t)d.RB * 4);                        // counters
  return off;
}

cudaError_t launch_decode(const ForwardArgs &a, cudaStream_t st, Launcher &L) {
  const DecTile d = dec_tile(a.M, a.K, a.n_sal, a.T);
  DecodeParams p;
  p.M = a.M; p.K = a.K; p.T = a.T; p.n_sal = a.n_sal; p.rank = a.rank; p.block = a.block;
  p.nkb = a.K / a.block;
  p.NR = d.NR; p.BK = d.BK; p.KT = d.KT; p.RB = d.RB; p.SE = d.SE; p.nq8box = d.nq8box;
  p.c = (float)sqrt(1.0 / (double)a.block);
  p.s4 = a.s4; p.sal_idx = a.sal_idx; p.s8 = a.s8; p.U = a.U; p.V = a.V;
  p.x = a.x; p.bias = a.bias; p.y = a.y; p.y_bf16 = a.y_bf16;
  char *ws = static_cast<char *>(a.workspace);
  size_t off = 0;
  auto take = [&](size_t b) { char *q = ws + off; off += (b + 255) & ~(size_t)255; return q; };
  p.xr16 = reinterpret_cast<__half *>(take((size_t)a.T * a.K * 2));
  p.xs16 = reinterpret_cast<__half *>(take((size_t)a.T * a.n_sal * 2 + 16));
  p.tp = reinterpret_cast<float *>(take((size_t)p.nkb * a.rank * a.T * 4));
  p.part = reinterpret_cast<float *>(take((size_t)p.KT * a.T * a.M * 4));
  p.counters = reinterpret_cast<unsigned int *>(take((size_t)p.RB * 4));

  CUtensorMap mq4, mq8, ms4, mu;
  if (encode_tmap_2d(&mq4, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q4, (uint64_t)a.K / 2, (uint64_t)a.M,
                     (uint64_t)a.K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // scale rows are K/32 bytes: a tensor map needs a multiple of 16, and the
  // box start (k0/64 elements) is aligned because k0 is a multiple of 1024
  p.s4_tma = (a.K % 512 == 0) && ((uintptr_t)a.s4 % 16 == 0);
  ms4 = mq4;
  if (p.s4_tma &&
      encode_tmap_2d(&ms4, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.s4, (uint64_t)a.K / 64,
                     (uint64_t)a.M, (uint64_t)a.K / 32, 16 * d.NR, 64,
                     CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
    p.s4_tma = 0;
  p.u_tma = a.rank > 0 && (a.rank % 8 == 0) && ((uintptr_t)a.U % 16 == 0);
  mu = mq4;
  if (p.u_tma &&
      encode_tmap_2d(&mu, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.U, (uint64_t)a.rank, (uint64_t)a.M,
                     (uint64_t)a.rank * 2, a.rank, 64, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
    p.u_tma = 0;
  if (a.n_sal > 0) {
    if (encode_tmap_2d(&mq8, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q8, (uint64_t)a.n_sal,
                       (uint64_t)a.M, (uint64_t)a.n_sal, 64, 64,
                       CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    mq8 = mq4;   // never used
  }
  cudaError_t e;
  const size_t vsm = (size_t)a.rank * (a.block + 8) * 2;
  if (a.block == 256)
    e = L.launch("dec_prologue", dec_prologue_kernel<256>, dim3(p.nkb), dim3(256), vsm, st, false, p);
  else
    e = L.launch("dec_prologue", dec_prologue_kernel<128>, dim3(p.nkb), dim3(128), vsm, st, false, p);
  if (e != cudaSuccess) return e;
  const size_t smem = dec_smem_bytes(d);
  if (a.T <= 8)
    return L.launch("dec_main", dec_main_kernel<1>, dim3(p.RB, p.KT), dim3(kDecThreads), smem, st,
                    true, mq4, mq8, ms4, mu, p);
  return L.launch("dec_main", dec_main_kernel<2>, dim3(p.RB, p.KT), dim3(kDecThreads), smem, st,
                  true, mq4, mq8, ms4, mu, p);
}

cudaError_t prepare_decode_kernels() {
  cudaError_t e;
  for (const void *f : {(const void *)dec_main_kernel<1>, (const void *)dec_main_kernel<2>,
                        (const void *)dec_prologue_kernel<256>, (const void *)dec_prologue_kernel<128>})
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
  if ((e = cudaFuncSetAttribute(dec_main_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                200 * 1024)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(dec_main_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                200 * 1024)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(dec_prologue_kernel<256>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 264 * 2)) !=
      cudaSuccess)
    return e;
  return cudaFuncSetAttribute(dec_prologue_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              64 * 136 * 2);
}

}  // namespace dvssq
