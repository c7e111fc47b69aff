// Prefill-shaped forward (many tokens) of the DV-SSQ layer on the 5th-
// generation tensor cores: the MiniCPM5-2B-Hadamard-GSQ card's runtime
// equation (§2) with the Spark card's INT8 salient tier, as ONE dense
// contraction over a concatenated reduction axis:
//
//   y[t][m] = sum_k A[m][k] * Xc[t][k] + bias[m]
//   A  = [ q4 . s4 (K cols) | q8 . s8 (n_sal, padded to 64) | U (r, padded to 64) ]
//   Xc = [ H x             | (H x)[sal_idx]                | V H x                ]
//
// pre_act   one CTA per 16 tokens builds Xc in FP16: fp32 Kronecker FWHT of
//           each Hadamard block, the salient gather, and t = V xr with
//           mma.sync (fp32 accumulation over all blocks).
// pre_mat   materialises A in FP16 once per call (the GPU counterpart of the
//           Spark card's materialize_weights), alongside pre_act: q4 . s4 is
//           exact in FP16 for scales in [2^-17, 8188]; q8 . s8 and U are
//           rounded once.
// pre_gemm  CTA tile 128 rows x BN tokens.  Warp 0 streams the A and Xc
//           tiles of each K stage by TMA (128B swizzle, no multicast); warp 1
//           issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM accumulator and
//           commits each stage back to the producer; warps 2-5 read TMEM
//           (tcgen05.ld) and write y.
#include "common.cuh"
#include "fwht_group.cuh"
#include "kernels.h"

namespace dvssq {

constexpr int kPreBM = 128;
constexpr int kPreStages = 4;
constexpr int kPreThreads = 192;

struct PrefillParams {
  int M, K, T, n_sal, salp, rank, Kc, nstages, nq4, nsal;
  float c;
  const uint8_t *q4;
  const uint16_t *s4;
  const int32_t *sal_idx;
  const int8_t *q8;
  const uint16_t *s8;
  const uint16_t *U;
  const uint16_t *V;
  const uint16_t *x;
  const uint16_t *bias;
  void *y;
  int y_bf16;
  __half *xc;      // [T][Kc]
  __half *a;       // [M][Kc]
  int nsplit;      // CTAs per 16-token group in pre_act, each a run of Hadamard blocks
  float *tpart;    // [nsplit][T][rank] t partials when nsplit > 1
  unsigned int *tdone;   // [T/16] finished splits per token group (zero at launch)
};

// ------------------------------------------------------------------ pre_act
// Dynamic shared memory of pre_act: FP16 block [16][B+8], FP16 V block
// [rank][B+8], sal_idx copy [n_sal], first salient entry of each Hadamard
// block [K/B + 1] (K/B <= 512).
static size_t pre_act_smem_bytes(int B, int rank, int n_sal) {
  return (size_t)16 * (B + 8) * 2 + (size_t)rank * (B + 8) * 2 + (size_t)n_sal * 4 + 513 * 4;
}

template <int B, int VPT>
__device__ __forceinline__ void pre_act_block(const PrefillParams &p, const int blk,
                                              const int split) {
  constexpr int P = B / 16;
  constexpr int NW = B / 32;
  __shared__ float scratch[16][GroupScratch<B>::kElems];
  extern __shared__ __align__(16) uint8_t dsm[];
  __half (*xh)[B + 8] = reinterpret_cast<__half (*)[B + 8]>(dsm);
  __half (*vh)[B + 8] = reinterpret_cast<__half (*)[B + 8]>(dsm + 16 * (B + 8) * 2);
  int *sidx = reinterpret_cast<int *>(dsm + 16 * (B + 8) * 2 + (size_t)p.rank * (B + 8) * 2);
  int *sblk = sidx + p.n_sal;        // first salient entry at or after column kb B

  const int tid = threadIdx.x, tok = tid / P, t = tid % P;
  const int t0 = blk * 16, gt = t0 + tok;
  const bool live = gt < p.T;
  const int nkb = p.K / B;
  // this CTA's run of Hadamard blocks
  const int kbA = (int)((long long)split * nkb / p.nsplit);
  const int kbB = (int)((long long)(split + 1) * nkb / p.nsplit);
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, tig = lane & 3;
  for (int e = tid; e < p.n_sal; e += B) sidx[e] = p.sal_idx[e];
  __syncthreads();
  // salient entries of block kb: [sblk[kb], sblk[kb + 1]) (sal_idx is ascending)
  for (int kb = tid; kb <= nkb; kb += B) {
    int lo = 0, hi = p.n_sal;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sidx[mid] < kb * B) lo = mid + 1; else hi = mid;
    }
    sblk[kb] = lo;
  }

  // t accumulators: n-tile (8 ranks) nt = warp + NW * j, j = 0, 1
  float tacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const int ntiles = (p.rank + 7) / 8;

  // the next block's x (registers) and V rows (registers, stored to vh at the
  // top of its iteration) are loaded one block ahead, so that their latency
  // overlaps the current block's work; VPT uint4 of V per thread cover the rank
  uint16_t xn[16];
  uint4 vn[VPT];
  auto fetch = [&](int kb) {
#pragma unroll
    for (int a = 0; a < 16; ++a)
      xn[a] = live ? p.x[(size_t)gt * p.K + (size_t)kb * B + P * a + t] : (uint16_t)0;
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int i = tid + u * B;
      const int rr = i / (B / 8), cc = i % (B / 8);
      vn[u] = rr < p.rank
                  ? *reinterpret_cast<const uint4 *>(p.V + (size_t)rr * p.K + (size_t)kb * B + cc * 8)
                  : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  if (kbA < kbB) fetch(kbA);
  for (int kb = kbA; kb < kbB; ++kb) {
    float v[16];
#pragma unroll
    for (int a = 0; a < 16; ++a) v[a] = bf16_bits_to_f32(xn[a]);
    // V block as FP16 (vh is free: the previous iteration ended with a barrier)
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int i = tid + u * B;
      const int rr = i / (B / 8), cc = i % (B / 8);
      if (rr < p.rank) {
        const uint32_t wv[4] = {vn[u].x, vn[u].y, vn[u].z, vn[u].w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          o[q] = pack_half2(__float2half_rn(bf16_bits_to_f32(wv[q] & 0xFFFFu)),
                            __float2half_rn(bf16_bits_to_f32(wv[q] >> 16)));
        *reinterpret_cast<uint4 *>(&vh[rr][cc * 8]) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    if (kb + 1 < kbB) fetch(kb + 1);
    fwht_group<B>(v, scratch[tok], t);
    uint32_t h[8];
#pragma unroll
    for (int j = 0; j < 16; j += 2)
      h[j / 2] = pack_half2(__float2half_rn(v[j] * p.c), __float2half_rn(v[j + 1] * p.c));
    *reinterpret_cast<uint4 *>(&xh[tok][16 * t]) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4 *>(&xh[tok][16 * t + 8]) = make_uint4(h[4], h[5], h[6], h[7]);
    if (live) {
      uint4 *dst = reinterpret_cast<uint4 *>(p.xc + (size_t)gt * p.Kc + (size_t)kb * B + 16 * t);
      dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
      dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
    }
    __syncthreads();
    // salient gather: the block's entries, consecutive lanes on consecutive
    // entries of one token (the FP16 block holds RN16 of the rotated values)
    {
      const int e_lo = sblk[kb], ne = sblk[kb + 1] - e_lo;
      for (int i = tid; i < ne * 16; i += B) {
        const int q = i / ne, e = e_lo + (i - q * ne);
        const int col = sidx[e] - kb * B;
        if (t0 + q < p.T && col >= 0 && col < B)
          p.xc[(size_t)(t0 + q) * p.Kc + p.K + e] = xh[q][col];
      }
    }
    // t += xr_block (16 x B) . V_block^T (B x 8) per n-tile of 8 ranks
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int nt = warp + NW * j;
      if (nt >= ntiles) break;
      const int n = 8 * nt + g;
#pragma unroll 4
      for (int k0 = 0; k0 < B; k0 += 16) {
        uint32_t a[4];
        a[0] = *reinterpret_cast<const uint32_t *>(&xh[g][k0 + 2 * tig]);
        a[1] = *reinterpret_cast<const uint32_t *>(&xh[g + 8][k0 + 2 * tig]);
        a[2] = *reinterpret_cast<const uint32_t *>(&xh[g][k0 + 2 * tig + 8]);
        a[3] = *reinterpret_cast<const uint32_t *>(&xh[g + 8][k0 + 2 * tig + 8]);
        const uint32_t b0 = n < p.rank ? *reinterpret_cast<const uint32_t *>(&vh[n][k0 + 2 * tig]) : 0u;
        const uint32_t b1 =
            n < p.rank ? *reinterpret_cast<const uint32_t *>(&vh[n][k0 + 2 * tig + 8]) : 0u;
        mma_16816(tacc[j], a, b0, b1, tacc[j]);
      }
    }
    __syncthreads();
  }
  // t: one split writes it directly; several write FP32 partials and the
  // last to finish adds them in split order
  if (p.nsplit > 1) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int nt = warp + NW * j;
      if (nt >= ntiles) break;
      const int n = 8 * nt + 2 * tig;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = g + 8 * (i >> 1), rr = n + (i & 1);
        if (t0 + q < p.T && rr < p.rank)
          p.tpart[((size_t)split * p.T + t0 + q) * p.rank + rr] = tacc[j][i];
      }
    }
    __shared__ unsigned int s_last;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&p.tdone[blk], 1u) == (unsigned int)(p.nsplit - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = tid; i < 16 * p.rank; i += B) {
      const int q = i / p.rank, rr = i - q * p.rank;
      if (t0 + q >= p.T) continue;
      float v = 0.0f;
      for (int sp = 0; sp < p.nsplit; ++sp)
        v += __ldcg(p.tpart + ((size_t)sp * p.T + t0 + q) * p.rank + rr);
      p.xc[(size_t)(t0 + q) * p.Kc + p.K + p.salp + rr] = __float2half_rn(v);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int nt = warp + NW * j;
      if (nt >= ntiles) break;
      const int n = 8 * nt + 2 * tig;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = g + 8 * (i >> 1), rr = n + (i & 1);
        if (t0 + q < p.T && rr < p.rank)
          p.xc[(size_t)(t0 + q) * p.Kc + p.K + p.salp + rr] = __float2half_rn(tacc[j][i]);
      }
    }
  }
  // the zero padding of the salient and low-rank sections
  const int npad1 = p.salp - p.n_sal, npad2 = 64 - p.rank;
  for (int i = tid; i < 16 * (npad1 + npad2); i += B) {
    const int q = i / (npad1 + npad2), j = i % (npad1 + npad2);
    if (t0 + q >= p.T) continue;
    const int col = j < npad1 ? p.K + p.n_sal + j : p.K + p.salp + p.rank + (j - npad1);
    p.xc[(size_t)(t0 + q) * p.Kc + col] = __float2half_rn(0.0f);
  }
}

// ------------------------------------------------------------------ pre_mat
// 8 nibbles (two's complement) of word w times scale s -> 4 FP16 pairs in
// column order (n0,n1), (n2,n3), (n4,n5), (n6,n7); exact for FP16-safe s.
__device__ __forceinline__ void dequant_q4_scaled(uint32_t w, __half2 s2, uint32_t out[4]) {
  const uint32_t u = w ^ 0x88888888u;
  const uint32_t magic = 0x64006400u;
  const __half2 sub_lo = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
  const __half2 mul_hi = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));
  const __half2 sub_hi = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));
  uint32_t l0 = (u & 0x000F000Fu) | magic;
  uint32_t h0 = (u & 0x00F000F0u) | magic;
  uint32_t l1 = ((u >> 8) & 0x000F000Fu) | magic;
  uint32_t h1 = ((u >> 8) & 0x00F000F0u) | magic;
  __half2 p0 = __hmul2(__hsub2(*reinterpret_cast<__half2 *>(&l0), sub_lo), s2);          // (n0,n4)
  __half2 p1 = __hmul2(__hfma2(*reinterpret_cast<__half2 *>(&h0), mul_hi, sub_hi), s2);   // (n1,n5)
  __half2 p2 = __hmul2(__hsub2(*reinterpret_cast<__half2 *>(&l1), sub_lo), s2);          // (n2,n6)
  __half2 p3 = __hmul2(__hfma2(*reinterpret_cast<__half2 *>(&h1), mul_hi, sub_hi), s2);   // (n3,n7)
  const uint32_t a = *reinterpret_cast<uint32_t *>(&p0), b = *reinterpret_cast<uint32_t *>(&p1);
  const uint32_t c = *reinterpret_cast<uint32_t *>(&p2), d = *reinterpret_cast<uint32_t *>(&p3);
  out[0] = __byte_perm(a, b, 0x5410);   // (n0, n1)
  out[1] = __byte_perm(c, d, 0x5410);   // (n2, n3)
  out[2] = __byte_perm(a, b, 0x7632);   // (n4, n5)
  out[3] = __byte_perm(c, d, 0x7632);   // (n6, n7)
}

// A[m][8 c .. 8 c + 7] for one (row, 8-column chunk) per thread, so that a
// warp writes 512 contiguous bytes: chunks of the first K/8 columns are
// q4 . s4, then q8 . s8 (n_sal padded to 64), then U (padded to 64 columns).
__device__ __forceinline__ void pre_mat_item(const PrefillParams &p, const long long item) {
  const int nc = p.Kc / 8;
  if (item >= (long long)p.M * nc) return;
  const int m = (int)(item / nc), ci = (int)(item - (long long)m * nc);
  const int kq = p.K / 8, ks = p.salp / 8;
  uint32_t h[4];
  if (ci < kq) {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(p.q4 + (size_t)m * (p.K / 2)) + ci);
    const __half sh = __float2half_rn(bf16_bits_to_f32(p.s4[(size_t)m * (p.K / 64) + ci / 8]));
    dequant_q4_scaled(w, __halves2half2(sh, sh), h);
  } else if (ci < kq + ks) {
    const int e0 = 8 * (ci - kq);
    const float s8f = bf16_bits_to_f32(p.s8[m]);
    uint2 raw = make_uint2(0u, 0u);
    if (e0 < p.n_sal)
      raw = __ldg(reinterpret_cast<const uint2 *>(p.q8 + (size_t)m * p.n_sal + e0));
    const uint32_t wv[2] = {raw.x, raw.y};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t w = wv[u];
      const float f0 = (float)(int8_t)(w & 0xFF) * s8f, f1 = (float)(int8_t)((w >> 8) & 0xFF) * s8f;
      const float f2 = (float)(int8_t)((w >> 16) & 0xFF) * s8f, f3 = (float)(int8_t)(w >> 24) * s8f;
      h[2 * u] = pack_half2(__float2half_rn(f0), __float2half_rn(f1));
      h[2 * u + 1] = pack_half2(__float2half_rn(f2), __float2half_rn(f3));
    }
  } else {
    const int r0 = 8 * (ci - kq - ks);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int ra = r0 + 2 * j, rb = ra + 1;
      const float u0 = ra < p.rank ? bf16_bits_to_f32(p.U[(size_t)m * p.rank + ra]) : 0.0f;
      const float u1 = rb < p.rank ? bf16_bits_to_f32(p.U[(size_t)m * p.rank + rb]) : 0.0f;
      h[j] = pack_half2(__float2half_rn(u0), __float2half_rn(u1));
    }
  }
  *reinterpret_cast<uint4 *>(p.a + (size_t)m * p.Kc + 8 * ci) = make_uint4(h[0], h[1], h[2], h[3]);
}

// pre_act (one CTA per 16 tokens) lets pre_mat launch at once (programmatic
// dependent launch), so the bandwidth-bound materialisation fills the SMs the
// latency-bound activation pass leaves idle.  pre_mat reads only the packed
// weights; it waits for pre_act only before it exits, so that its completion
// (which orders the GEMM) implies pre_act's.
template <int B, int VPT>
__global__ void __launch_bounds__(B, 768 / B) pre_act_kernel(PrefillParams p) {
  pdl_launch_dependents();
  pre_act_block<B, VPT>(p, blockIdx.x, blockIdx.y);
}

__global__ void __launch_bounds__(256) pre_mat_kernel(PrefillParams p, long long items) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < items;
       i += (long long)gridDim.x * blockDim.x)
    pre_mat_item(p, i);
  pdl_wait();
}

// ----------------------------------------------------------------- pre_gemm
// Persistent: one CTA per SM walks output tiles, token tile fastest: a wave
// of CTAs shares a few row tiles of A (each read from DRAM once) and all the
// activation tiles, which are small enough to stay in L2 across waves.  TMEM
// holds two accumulators of BN columns: the MMA warp fills one while the
// epilogue warps drain the other (acc_full / acc_empty barriers).
template <int BN>
__global__ void __launch_bounds__(kPreThreads, 1) pre_gemm_kernel(
    const __grid_constant__ CUtensorMap ma, const __grid_constant__ CUtensorMap mxc,
    PrefillParams p, int nmt, int ntiles) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  constexpr int A_STAGE = kPreBM * 128;
  constexpr int B_STAGE = BN * 128;
  const int ntt = ntiles / nmt;      // token tiles
  uint8_t *sa = base;
  uint8_t *sb = base + kPreStages * A_STAGE;
  uint64_t *full = reinterpret_cast<uint64_t *>(sb + kPreStages * B_STAGE);
  uint64_t *empty = full + kPreStages;
  uint64_t *acc_full = empty + kPreStages;       // [2]
  uint64_t *acc_empty = acc_full + 2;            // [2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = p.nstages;

  if (tid == 0) {
    for (int s = 0; s < kPreStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ---------------- operand producer (TMA: weights and activations) ----------------
    if (lane == 0) {
      prefetch_tensormap(&ma);
      prefetch_tensormap(&mxc);
      long long gs = 0;                           // stage counter over all tiles
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int m0 = (tile / ntt) * kPreBM, n0 = (tile % ntt) * BN;
        for (int s = 0; s < S && ok; ++s, ++gs) {
          const int slot = (int)(gs % kPreStages);
          const uint32_t round = (uint32_t)(gs / kPreStages);
          if (!mbar_wait(&empty[slot], (round & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[slot], A_STAGE + B_STAGE);
          tma_load_2d(sa + slot * A_STAGE, &ma, 64 * s, m0, &full[slot]);
          tma_load_2d(sb + slot * B_STAGE, &mxc, 64 * s, n0, &full[slot]);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------- MMA issuer -----------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kPreBM, BN);
      long long gs = 0;
      int li = 0;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++li) {
        const int ab = li & 1;
        if (!mbar_wait(&acc_empty[ab], ((li >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(ab * BN);
        for (int s = 0; s < S && ok; ++s, ++gs) {
          const int slot = (int)(gs % kPreStages);
          const uint32_t round = (uint32_t)(gs / kPreStages);
          if (!mbar_wait(&full[slot], round & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sa + slot * A_STAGE), b0 = smem_u32(sb + slot * B_STAGE);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_f16(acc, umma_desc_sw128(a0 + 32 * k), umma_desc_sw128(b0 + 32 * k), idesc,
                       (s > 0 || k > 0) ? 1u : 0u);
          tc_commit(&empty[slot]);
        }
        tc_commit(&acc_full[ab]);
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int quarter = warp & 3;
    int li = 0;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++li) {
      const int ab = li & 1;
      const int m0 = (tile / ntt) * kPreBM, n0 = (tile % ntt) * BN;
      if (!mbar_wait(&acc_full[ab], (li >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const int row = m0 + 32 * quarter + lane;
      const float bv = (p.bias != nullptr && row < p.M) ? bf16_bits_to_f32(p.bias[row]) : 0.0f;
#pragma unroll 1
      for (int c = 0; c < BN / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(ab * BN) + 16 * c, r);
        tmem_ld_wait();
        if (row < p.M) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = n0 + 16 * c + j;
            if (tok < p.T) {
              const float v = __uint_as_float(r[j]) + bv;
              // streaming stores (evict-first): the output is written once and
              // must not push the A and activation tiles out of L2
              if (p.y_bf16)
                __stcs(reinterpret_cast<unsigned short *>(p.y) + (size_t)tok * p.M + row,
                       (unsigned short)f32_to_bf16_rn_bits(v));
              else
                __stcs(reinterpret_cast<float *>(p.y) + (size_t)tok * p.M + row, v);
            }
          }
        }
      }
      // this accumulator may be overwritten by the tile after next
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// ---------------------------------------------------------------- host ---
static int pre_bn(int T) { return T > 128 ? 256 : (T > 64 ? 128 : 64); }

static size_t pre_smem_bytes(int BN) {
  return 1024 + (size_t)kPreStages * (kPreBM * 128 + BN * 128) + 256;   // + barriers, TMEM slot
}

// CTAs per 16-token group in pre_act: enough for about four resident CTAs
// on each of B200's 148 SMs, each a run of at least one Hadamard block.  A
// host-side constant (no device query), so the workspace size stays a pure
// function of the shape; any split count gives the same result.
constexpr int kPreActSlots = 4 * 148;
static int pre_act_splits(int nkb, int T) {
  const int ntg = (T + 15) / 16;
  const int want = (kPreActSlots + ntg - 1) / ntg;
  return std::max(1, std::min(nkb, want));
}

size_t prefill_workspace_bytes(int M, int K, int block, int n_sal, int rank, int T) {
  (void)block; (void)rank;
  const int salp = (n_sal + 63) / 64 * 64;
  const size_t Kc = (size_t)K + salp + 64;
  // Xc [T][Kc] and the materialised A [M][Kc], FP16; pre_act's t partials
  // [nsplit][T][rank] and per-16-token counters
  const int ns = pre_act_splits(K / block, T);
  return (((size_t)T * Kc * 2 + 255) & ~(size_t)255) + (((size_t)M * Kc * 2 + 255) & ~(size_t)255) +
         (((size_t)ns * T * 64 * 4 + 255) & ~(size_t)255) + (((size_t)(T + 15) / 16 * 4 + 255) & ~(size_t)255);
}

cudaError_t launch_prefill(const ForwardArgs &a, cudaStream_t st, Launcher &L) {
  PrefillParams p;
  p.M = a.M; p.K = a.K; p.T = a.T; p.n_sal = a.n_sal; p.rank = a.rank;
  p.salp = (a.n_sal + 63) / 64 * 64;
  p.Kc = a.K + p.salp + 64;
  p.nq4 = a.K / 64;
  p.nsal = p.salp / 64;
  p.nstages = p.nq4 + p.nsal + (a.rank > 0 ? 1 : 0);
  p.c = (float)sqrt(1.0 / (double)a.block);
  p.q4 = a.q4; p.s4 = a.s4; p.sal_idx = a.sal_idx; p.q8 = a.q8; p.s8 = a.s8;
  p.U = a.U; p.V = a.V; p.x = a.x; p.bias = a.bias; p.y = a.y; p.y_bf16 = a.y_bf16;
  p.xc = reinterpret_cast<__half *>(a.workspace);
  p.a = reinterpret_cast<__half *>(static_cast<char *>(a.workspace) +
                                   (((size_t)a.T * p.Kc * 2 + 255) & ~(size_t)255));

  {
    const size_t off_tp = (((size_t)a.T * p.Kc * 2 + 255) & ~(size_t)255) +
                          (((size_t)a.M * p.Kc * 2 + 255) & ~(size_t)255);
    p.nsplit = pre_act_splits(a.K / a.block, a.T);
    p.tpart = reinterpret_cast<float *>(static_cast<char *>(a.workspace) + off_tp);
    p.tdone = reinterpret_cast<unsigned int *>(
        static_cast<char *>(a.workspace) + off_tp +
        (((size_t)p.nsplit * a.T * 64 * 4 + 255) & ~(size_t)255));
  }
  const size_t act_smem = pre_act_smem_bytes(a.block, a.rank, a.n_sal);
  cudaError_t e;
  if (p.nsplit > 1) {
    e = cudaMemsetAsync(p.tdone, 0, (size_t)(a.T + 15) / 16 * sizeof(unsigned int), st);
    if (e != cudaSuccess) return e;
  }
  const dim3 ga((a.T + 15) / 16, p.nsplit);
#define DVSSQ_PRE_ACT(BB, VV) \
  L.launch("pre_act", pre_act_kernel<BB, VV>, ga, dim3(BB), act_smem, st, false, p)
  if (a.block == 256)
    e = a.rank <= 16 ? DVSSQ_PRE_ACT(256, 2) : a.rank <= 32 ? DVSSQ_PRE_ACT(256, 4)
                                                            : DVSSQ_PRE_ACT(256, 8);
  else
    e = a.rank <= 16 ? DVSSQ_PRE_ACT(128, 2) : a.rank <= 32 ? DVSSQ_PRE_ACT(128, 4)
                                                            : DVSSQ_PRE_ACT(128, 8);
#undef DVSSQ_PRE_ACT
  if (e != cudaSuccess) return e;
  const long long items = (long long)a.M * (p.Kc / 8);
  const long long mat_blocks = std::min<long long>((items + 255) / 256, (long long)sm_count() * 8);
  e = L.launch("pre_mat", pre_mat_kernel, dim3((unsigned)mat_blocks), dim3(256), 0, st, true, p,
               items);
  if (e != cudaSuccess) return e;


  CUtensorMap mxc, ma;
  const int BN = pre_bn(a.T);
  if (encode_tmap_2d(&mxc, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.xc, (uint64_t)p.Kc, (uint64_t)a.T,
                     (uint64_t)p.Kc * 2, 64, (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tmap_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, p.a, (uint64_t)p.Kc, (uint64_t)a.M,
                     (uint64_t)p.Kc * 2, 64, kPreBM, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int nmt = (a.M + kPreBM - 1) / kPreBM;
  const int ntiles = nmt * ((a.T + BN - 1) / BN);
  const dim3 gg((unsigned)std::min(ntiles, sm_count()));
  const size_t smem = pre_smem_bytes(BN);
  if (BN == 256)
    return L.launch("pre_gemm", pre_gemm_kernel<256>, gg, dim3(kPreThreads), smem, st, false, ma,
                    mxc, p, nmt, ntiles);
  if (BN == 128)
    return L.launch("pre_gemm", pre_gemm_kernel<128>, gg, dim3(kPreThreads), smem, st, false, ma,
                    mxc, p, nmt, ntiles);
  return L.launch("pre_gemm", pre_gemm_kernel<64>, gg, dim3(kPreThreads), smem, st, false, ma, mxc,
                  p, nmt, ntiles);
}

cudaError_t prepare_prefill_kernels() {
  cudaError_t e;
  const void *acts[] = {(const void *)pre_act_kernel<256, 2>, (const void *)pre_act_kernel<256, 4>,
                        (const void *)pre_act_kernel<256, 8>, (const void *)pre_act_kernel<128, 2>,
                        (const void *)pre_act_kernel<128, 4>, (const void *)pre_act_kernel<128, 8>};
  for (int i = 0; i < 6; ++i) {
    if ((e = cudaFuncSetAttribute(acts[i], cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(acts[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)pre_act_smem_bytes(i < 3 ? 256 : 128, 64, kMaxSalient))) !=
        cudaSuccess)
      return e;
  }
  e = cudaFuncSetAttribute(pre_gemm_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)pre_smem_bytes(256));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(pre_gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)pre_smem_bytes(128));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(pre_gemm_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)pre_smem_bytes(64));
  if (e != cudaSuccess) return e;
  return cudaSuccess;
}

}  // namespace dvssq
