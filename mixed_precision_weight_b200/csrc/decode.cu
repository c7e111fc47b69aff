// Decode-shaped forward (T <= 16 tokens) of the DV-SSQ layer: the runtime
// equation of the MiniCPM5-2B-Hadamard-GSQ card (§2, Y = X What^T + (X B^T)
// A^T) with the Spark card's INT8 salient tier, on the packed form.
//
// Two launches, chained by programmatic dependent launch:
//   dec_prologue  one CTA per Hadamard block: xr = H_b x in fp32 (16-thread
//                 Kronecker FWHT), written as FP16 in the GEMV's k-order; the
//                 salient entries xs = xr[sal_idx]; per-block partials of
//                 t = V xr; zeroes the split-K arrival counters.
//   dec_main      CTA tile = 64 rows x 1024 columns.  TMA brings the whole
//                 q4 tile (128B-swizzled) and the CTA's q8 slice (64B-
//                 swizzled) into shared memory at once, before waiting on the
//                 prologue, so the weight stream overlaps it.  Each warp owns
//                 128 columns of all 64 rows: nibbles -> exact FP16 codes in
//                 registers -> mma.sync m16n8k16 (FP32 accumulation) per
//                 64-column group, then acc += s4 * group sum in FP32.  The
//                 salient tier accumulates q8 codes separately and is scaled
//                 by s8.  Warps reduce in shared memory, CTAs write split-K
//                 partials, and the last CTA of each row block sums them in
//                 k order, adds U t and the bias, and writes y.
#include "common.cuh"
#include "fwht_group.cuh"
#include "kernels.h"

namespace dvssq {

constexpr int kDecBM = 64;
constexpr int kDecBK = 1024;
constexpr int kDecThreads = 256;
constexpr int kDecQ4Box = 64 * 128;      // bytes of one q4 box (64 rows x 256 cols)
constexpr int kDecQ8Box = 64 * 64;       // bytes of one q8 box (64 rows x 64 entries)

struct DecodeParams {
  int M, K, T, n_sal, rank, nkb, KT, RB, SE, nq8box;
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

// Position i of each 16-column segment of xr16 holds column kPerm[i]: the
// order in which nibble pairs come out of the dequantiser (see dequant_q4).
__constant__ int kPerm[16] = {0, 4, 1, 5, 2, 6, 3, 7, 8, 12, 9, 13, 10, 14, 11, 15};

// ------------------------------------------------------------- prologue ---
template <int B>
__global__ void __launch_bounds__(B) dec_prologue_kernel(DecodeParams p) {
  pdl_launch_dependents();
  constexpr int P = B / 16;
  __shared__ float scratch[16][GroupScratch<B>::kElems];
  __shared__ float xr[16][B + 1];
  __shared__ __align__(16) uint16_t vs[16][B + 8];
  __shared__ int s_cnt[2];

  const int kb = blockIdx.x, tid = threadIdx.x;
  const int tok = tid / P, t = tid % P;
  if (kb == 0)
    for (int i = tid; i < p.RB; i += B) p.counters[i] = 0u;
  if (tid < 2) s_cnt[tid] = 0;

  float v[16];
  const bool live = tok < p.T;
#pragma unroll
  for (int a = 0; a < 16; ++a)
    v[a] = live ? bf16_bits_to_f32(p.x[(size_t)tok * p.K + (size_t)kb * B + P * a + t]) : 0.0f;
  fwht_group<B>(v, scratch[tok], t);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    v[j] *= p.c;
    xr[tok][16 * t + j] = v[j];
  }
  if (live) {
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      h[i] = pack_half2(__float2half_rn(v[kPerm[2 * i]]), __float2half_rn(v[kPerm[2 * i + 1]]));
    uint4 *dst = reinterpret_cast<uint4 *>(p.xr16 + (size_t)tok * p.K + (size_t)kb * B + 16 * t);
    dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
    dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
  }
  // salient entries whose rotated column falls in this block
  int lo = 0, hi = 0;
  for (int e = tid; e < p.n_sal; e += B) {
    const int s = p.sal_idx[e];
    lo += s < kb * B;
    hi += s < (kb + 1) * B;
  }
  __syncthreads();
  if (lo) atomicAdd(&s_cnt[0], lo);
  if (hi) atomicAdd(&s_cnt[1], hi);
  __syncthreads();
  const int e_lo = s_cnt[0], e_hi = s_cnt[1];
  for (int e = e_lo + tid; e < e_hi; e += B) {
    const int col = p.sal_idx[e] - kb * B;
    if (col < 0 || col >= B) continue;   // sal_idx must be sorted; ignore otherwise
    for (int q = 0; q < p.T; ++q)
      p.xs16[(size_t)q * p.n_sal + e] = __float2half_rn(xr[q][col]);
  }
  // partials of t = V xr over this block, 16 rows of V at a time
  for (int r0 = 0; r0 < p.rank; r0 += 16) {
    const int nr = min(16, p.rank - r0);
    __syncthreads();
    for (int i = tid; i < nr * (B / 8); i += B) {
      const int rr = i / (B / 8), cc = i % (B / 8);
      *reinterpret_cast<uint4 *>(&vs[rr][cc * 8]) = *reinterpret_cast<const uint4 *>(
          p.V + (size_t)(r0 + rr) * p.K + (size_t)kb * B + cc * 8);
    }
    __syncthreads();
    for (int pr = tid; pr < nr * p.T; pr += B) {
      const int rr = pr / p.T, q = pr % p.T;
      float acc = 0.0f;
#pragma unroll 8
      for (int j = 0; j < B; ++j) acc = fmaf(bf16_bits_to_f32(vs[rr][j]), xr[q][j], acc);
      p.tp[((size_t)kb * p.rank + r0 + rr) * p.T + q] = acc;
    }
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

__global__ void __launch_bounds__(kDecThreads) dec_main_kernel(
    const __grid_constant__ CUtensorMap mq4, const __grid_constant__ CUtensorMap mq8,
    DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *sq4 = base;                                        // 4 boxes, 32 KB
  uint8_t *sq8 = base + 4 * kDecQ4Box;                        // nq8box boxes
  uint16_t *ss4 = reinterpret_cast<uint16_t *>(sq8 + p.nq8box * kDecQ8Box);   // 64 x 16
  float *tfin = reinterpret_cast<float *>(ss4 + kDecBM * 16);                 // rank x T
  uint64_t *bars = reinterpret_cast<uint64_t *>(tfin + 64 * 16);              // 5
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int rb = blockIdx.x, kt = blockIdx.y;
  const int m0 = rb * kDecBM, k0 = kt * kDecBK, e0 = kt * p.SE;
  const int nsal_cta = max(0, min(p.SE, p.n_sal - e0));

  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    prefetch_tensormap(&mq4);
#pragma unroll
    for (int box = 0; box < 4; ++box) {
      if (k0 + 256 * box < p.K) {
        mbar_arrive_expect_tx(&bars[box], kDecQ4Box);
        tma_load_2d(sq4 + box * kDecQ4Box, &mq4, (k0 + 256 * box) / 2, m0, &bars[box]);
      }
    }
    if (nsal_cta > 0) {
      const int nb = (nsal_cta + 63) / 64;
      mbar_arrive_expect_tx(&bars[4], nb * kDecQ8Box);
      for (int i = 0; i < nb; ++i)
        tma_load_2d(sq8 + i * kDecQ8Box, &mq8, e0 + 64 * i, m0, &bars[4]);
    }
  }
  // group scales of the tile (independent of the prologue)
  const int KG = p.K / 64;
  for (int i = tid; i < kDecBM * 16; i += kDecThreads) {
    const int r = i >> 4, gi = i & 15;
    const int row = m0 + r, gcol = k0 / 64 + gi;
    ss4[i] = (row < p.M && gcol < KG) ? p.s4[(size_t)row * KG + gcol] : (uint16_t)0;
  }

  pdl_wait();   // xr16, xs16, tp and the counters come from the prologue

  const int NT = (p.T + 7) >> 3;
  const int kw = k0 + 128 * warp;                 // this warp's first column
  const bool have = kw < p.K;
  uint32_t bq[2][2][8];
#pragma unroll
  for (int gi = 0; gi < 2; ++gi)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int tok = g + 8 * nt;
      const int kc = kw + 64 * gi + 16 * tig;
      if (nt < NT && tok < p.T && kc < p.K) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.xr16 + (size_t)tok * p.K + kc);
        uint4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
        bq[gi][nt][0] = x0.x; bq[gi][nt][1] = x0.y; bq[gi][nt][2] = x0.z; bq[gi][nt][3] = x0.w;
        bq[gi][nt][4] = x1.x; bq[gi][nt][5] = x1.y; bq[gi][nt][6] = x1.z; bq[gi][nt][7] = x1.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) bq[gi][nt][i] = 0u;
      }
    }
  __syncthreads();   // ss4 complete

  float acc[4][2][4];
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[rt][nt][i] = 0.0f;

  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
  const int box = warp >> 1, half = warp & 1;
  if (have && mbar_wait(&bars[box], 0)) {
    const uint8_t *bx = sq4 + box * kDecQ4Box;
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
      const int chunk = 4 * half + 2 * gi + (tig >> 1);
      const int sgrp = 2 * warp + gi;
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
        const float slo = bf16_bits_to_f32(ss4[rlo * 16 + sgrp]);
        const float shi = bf16_bits_to_f32(ss4[(rlo + 8) * 16 + sgrp]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          if (nt >= NT) break;
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

  // salient INT8 tier: k16 steps of the CTA's salient slice, round robin
  if (nsal_cta > 0) {
    float acc8[4][2][4];
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc8[rt][nt][i] = 0.0f;
    bool any = false;
    const int nsteps = nsal_cta / 16;
    if (warp < nsteps && mbar_wait(&bars[4], 0)) {
      for (int st = warp; st < nsteps; st += 8) {
        any = true;
        const int e = e0 + 16 * st;
        uint32_t b01[2], b23[2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int tok = g + 8 * nt;
          if (nt < NT && tok < p.T) {
            const uint2 xv =
                __ldcg(reinterpret_cast<const uint2 *>(p.xs16 + (size_t)tok * p.n_sal + e + 4 * tig));
            b01[nt] = xv.x;
            b23[nt] = xv.y;
          } else {
            b01[nt] = 0u;
            b23[nt] = 0u;
          }
        }
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
          for (int nt = 0; nt < 2; ++nt) {
            if (nt >= NT) break;
            mma_16816(acc8[rt][nt], a, b01[nt], b23[nt], acc8[rt][nt]);
          }
        }
      }
    }
    if (any) {
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        const int rlo = m0 + 16 * rt + g, rhi = rlo + 8;
        const float s8lo = rlo < p.M ? bf16_bits_to_f32(p.s8[rlo]) : 0.0f;
        const float s8hi = rhi < p.M ? bf16_bits_to_f32(p.s8[rhi]) : 0.0f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          acc[rt][nt][0] = fmaf(s8lo, acc8[rt][nt][0], acc[rt][nt][0]);
          acc[rt][nt][1] = fmaf(s8lo, acc8[rt][nt][1], acc[rt][nt][1]);
          acc[rt][nt][2] = fmaf(s8hi, acc8[rt][nt][2], acc[rt][nt][2]);
          acc[rt][nt][3] = fmaf(s8hi, acc8[rt][nt][3], acc[rt][nt][3]);
        }
      }
    }
  }

  // reduce the 8 warps' k slices in shared memory (reusing the q4 boxes)
  __syncthreads();
  float *red = reinterpret_cast<float *>(base);      // [8][64][16]
#pragma unroll
  for (int rt = 0; rt < 4; ++rt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int rlo = 16 * rt + g, tok = 2 * tig + 8 * nt;
      red[(warp * 64 + rlo) * 16 + tok] = acc[rt][nt][0];
      red[(warp * 64 + rlo) * 16 + tok + 1] = acc[rt][nt][1];
      red[(warp * 64 + rlo + 8) * 16 + tok] = acc[rt][nt][2];
      red[(warp * 64 + rlo + 8) * 16 + tok + 1] = acc[rt][nt][3];
    }
  __syncthreads();
  for (int i = tid; i < kDecBM * 16; i += kDecThreads) {
    const int tok = i >> 6, r = i & 63;
    if (tok >= p.T || m0 + r >= p.M) continue;
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[(w * 64 + r) * 16 + tok];
    p.part[((size_t)kt * p.T + tok) * p.M + m0 + r] = v;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.counters[rb], 1u) == (unsigned)(p.KT - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // last CTA of this row block: t = sum over blocks of the prologue partials
  for (int i = tid; i < p.rank * p.T; i += kDecThreads) {
    float s = 0.0f;
    for (int kb = 0; kb < p.nkb; ++kb) s += __ldcg(&p.tp[(size_t)kb * p.rank * p.T + i]);
    tfin[i] = s;
  }
  __syncthreads();
  for (int i = tid; i < kDecBM * p.T; i += kDecThreads) {
    const int tok = i >> 6, r = i & 63, m = m0 + r;
    if (m >= p.M) continue;
    float v = 0.0f;
    for (int k = 0; k < p.KT; ++k) v += __ldcg(&p.part[((size_t)k * p.T + tok) * p.M + m]);
    for (int rr = 0; rr < p.rank; ++rr)
      v = fmaf(bf16_bits_to_f32(p.U[(size_t)m * p.rank + rr]), tfin[rr * p.T + tok], v);
    if (p.bias) v += bf16_bits_to_f32(p.bias[m]);
    if (p.y_bf16)
      reinterpret_cast<uint16_t *>(p.y)[(size_t)tok * p.M + m] = f32_to_bf16_rn_bits(v);
    else
      reinterpret_cast<float *>(p.y)[(size_t)tok * p.M + m] = v;
  }
}

// ---------------------------------------------------------------- host ---
static int dec_salient_span(int n_sal, int KT) {
  // salient entries per CTA, a multiple of 64 (one q8 box)
  const int boxes = (n_sal + 63) / 64;
  return 64 * ((boxes + KT - 1) / KT);
}

static size_t dec_smem_bytes(int nq8box, int rank, int T) {
  (void)rank;
  (void)T;
  return 1024 + 4 * kDecQ4Box + (size_t)nq8box * kDecQ8Box + kDecBM * 16 * 2 + 64 * 16 * 4 + 64;
}

size_t decode_workspace_bytes(int M, int K, int block, int n_sal, int rank, int T) {
  const int KT = (K + kDecBK - 1) / kDecBK, RB = (M + kDecBM - 1) / kDecBM;
  size_t off = 0;
  auto take = [&](size_t b) { off += (b + 255) & ~(size_t)255; };
  take((size_t)T * K * 2);                       // xr16
  take((size_t)T * n_sal * 2 + 16);              // xs16
  take((size_t)(K / block) * rank * T * 4);      // tp
  take((size_t)KT * T * M * 4);                  // split-K partials
  take((size_t)RB * 4);                          // counters
  return off;
}

cudaError_t launch_decode(const ForwardArgs &a, cudaStream_t st, Launcher &L) {
  DecodeParams p;
  p.M = a.M; p.K = a.K; p.T = a.T; p.n_sal = a.n_sal; p.rank = a.rank;
  p.nkb = a.K / a.block;
  p.KT = (a.K + kDecBK - 1) / kDecBK;
  p.RB = (a.M + kDecBM - 1) / kDecBM;
  p.SE = a.n_sal > 0 ? dec_salient_span(a.n_sal, p.KT) : 0;
  p.nq8box = p.SE / 64;
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

  CUtensorMap mq4, mq8;
  if (encode_tmap_2d(&mq4, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q4, (uint64_t)a.K / 2, (uint64_t)a.M,
                     (uint64_t)a.K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (a.n_sal > 0) {
    if (encode_tmap_2d(&mq8, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q8, (uint64_t)a.n_sal,
                       (uint64_t)a.M, (uint64_t)a.n_sal, 64, 64,
                       CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    mq8 = mq4;   // never used
  }
  cudaError_t e;
  if (a.block == 256)
    e = L.launch("dec_prologue", dec_prologue_kernel<256>, dim3(p.nkb), dim3(256), 0, st, false, p);
  else
    e = L.launch("dec_prologue", dec_prologue_kernel<128>, dim3(p.nkb), dim3(128), 0, st, false, p);
  if (e != cudaSuccess) return e;
  const size_t smem = dec_smem_bytes(p.nq8box, a.rank, a.T);
  return L.launch("dec_main", dec_main_kernel, dim3(p.RB, p.KT), dim3(kDecThreads), smem, st, true,
                  mq4, mq8, p);
}

cudaError_t prepare_decode_kernels() {
  return cudaFuncSetAttribute(dec_main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              200 * 1024);
}

}  // namespace dvssq
