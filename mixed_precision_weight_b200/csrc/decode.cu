// Decode-shaped forward (T <= 16 tokens) of the DV-SSQ layer: the runtime
// equation of the MiniCPM5-2B-Hadamard-GSQ card (§2, Y = X What^T + (X B^T)
// A^T) with the Spark card's INT8 salient tier, on the packed form.
//
// The layer is cut into work units of 16 rows x one 256-column slab (128
// bytes of nibbles per row).  Units are numbered slab-major and split into
// one contiguous, equal share per CTA (one CTA per SM), so every SM streams
// the same number of weight bytes.
//
// dec_main (programmatic dependent launch), warp 0 a producer, warps 1..15
// consumers that never wait behind it:
//   before the dependency wait - reads only the packed weights.  The
//     producer issues by TMA the V rows of the slab whose t share the CTA
//     writes, then every unit's q4 box (16 x 128 B, 128B swizzle) and s4
//     box.  The consumers find each slab's salient entries (a two-round
//     parallel search of sal_idx), lay out the INT8 chunks (16 entries each)
//     unit by unit and hand the layout to the producer through an mbarrier;
//     the producer stages the chunks of the units that fit in the free
//     shared memory, in unit order, and exits.  Units past that budget read
//     their chunks from global memory (L2).
//   after the wait - the CTA rotates x for its (at most kDecMaxSlabs) slabs
//     itself (16-thread Kronecker FWHT, fp32), stores it as FP16 in the
//     GEMV's k-order, scatters the salient entries, and forms per-group
//     bias terms.  The owned slab's t share (V x_rot over 256 columns) runs
//     on the tensor cores, its k range split over the warps and the warps'
//     pieces added in warp order.  Warps then take units round-robin:
//     nibbles become FP16 1024+u (even columns) or 1024+16u (odd columns,
//     whose activations are stored pre-divided by 16) with one LOP3 each;
//     the MMA chain of a 64-column group starts from minus the group's bias
//     term, so its sum is the exact-code dot product; acc += s4 * group sum.
//     The salient chunks run the same way (1152 + q) and are scaled by s8.
//     Each unit writes its 16 x T partial for its slab.
// dec_tail: y = sum over slabs of the partials (slab order, deterministic)
//   + U t + bias, in FP32, optionally rounded to BF16.
#include "common.cuh"
#include "fwht_group.cuh"
#include "kernels.h"

#include <algorithm>
#include <mutex>
#include <vector>

namespace dvssq {

constexpr int kSlab = 256;                   // rotated columns per slab
constexpr int kUnitRows = 16;                // rows per work unit
constexpr int kDecWarps = 16;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecCons = kDecWarps - 1;        // consumer warps (warp 0 issues the weight stream)
constexpr int kDecConsThreads = 32 * kDecCons;
constexpr int kDecNV = (64 + kDecCons - 1) / kDecCons;   // rank rows per consumer warp (rank <= 64)
constexpr int kDecMaxUnits = 48;             // units per CTA staged at once
constexpr int kDecMaxSlabs = 4;              // distinct slabs per CTA
constexpr int kQ4Unit = kUnitRows * 128;     // one q4 box: 16 rows x 128 B
constexpr int kS4Unit = kUnitRows * 16;      // one s4 box: 16 rows x 8 scales
constexpr int kQ8Chunk = kUnitRows * 16;     // one q8 box: 16 rows x 16 entries
constexpr int kXRow = kSlab + 8;             // FP16 per token row of x_rot (padded)
constexpr int kXsRow = 17 * 16 + 8;          // FP16 per token row of the salient x
constexpr int kSamples = 512;                // sal_idx samples of the search
constexpr int kTailThreads = 256;
constexpr int kSmemLimit = 232448;           // opt-in shared memory per CTA (227 KB)

// Shared-memory layout of dec_main: byte offsets from the 1024-aligned base.
struct DecLayout {
  int q4, s4, q8, xq, xs, corr, c8, s8, colpos, samp, scr, meta, bars, vs, total;
};

// Barrier among the consumer warps only (the producer warp leaves early).
__device__ __forceinline__ void dec_consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kDecConsThreads) : "memory");
}

// Tiles 4i..4i+3 of one slab whose units all lie in the CTA's range travel
// as one q4 box (and one s4 box) that lands exactly where four single-unit
// boxes would.  Returns the index within the CTA of the quad's first unit,
// or -1 for a unit staged on its own.
__device__ __forceinline__ int quad_lead(int u, int u0, int u1, int ntile, int quad) {
  if (!quad) return -1;
  const int s = u / ntile, tq = (u - s * ntile) & ~3;
  const int uq = s * ntile + tq;
  return (tq + 3 < ntile && uq >= u0 && uq + 3 < u1) ? uq - u0 : -1;
}

struct DecodeParams {
  int M, K, T, n_sal, rank, block;
  int nslab, ntile, units, grid, upc_max, ns_max, ntok, nscr;
  int q8_budget, s4_tma;
  int quad;       // four consecutive tiles of a slab may travel as one box
  float c;
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
  float *part;    // [slice][T][M]
  float *tpart;   // [nslab][rank][T]
  int nslices;    // partial slices dec_tail sums for every output
  DecLayout L;
};

// Position i of each 16-column segment of the FP16 x_rot holds column
// perm16(i): the order in which nibble pairs come out of dequant_q4_biased,
// i.e. {0,4,1,5, 2,6,3,7, 8,12,9,13, 10,14,11,15}.
__host__ __device__ constexpr int perm16(int i) {
  return (i & 8) | ((i & 1) << 2) | ((i >> 1) & 3);
}
__host__ __device__ constexpr int inv_perm16(int j) {
  return (j & 8) | ((j & 3) << 1) | ((j >> 2) & 1);
}

// Per bit: b ? (c ? ~a : a) : c.  With b a nibble mask and c holding the
// bias bit (inside the mask) and the FP16 exponent pattern (outside it), one
// instruction flips the sign bit of each selected nibble and splices it into
// the mantissa of an FP16 1024.
__device__ __forceinline__ uint32_t lop3_splice(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 8 two's-complement nibbles (columns c0..c7) -> FP16 pairs (c0,c4), (c1,c5),
// (c2,c6), (c3,c7) holding 1024 + u for even columns and 1024 + 16u for odd
// ones, u = q + 8 in [0, 15].  Exact.
__device__ __forceinline__ void dequant_q4_biased(uint32_t w, uint32_t out[4]) {
  const uint32_t w8 = w >> 8;
  out[0] = lop3_splice(w, 0x000F000Fu, 0x64086408u);
  out[1] = lop3_splice(w, 0x00F000F0u, 0x64806480u);
  out[2] = lop3_splice(w8, 0x000F000Fu, 0x64086408u);
  out[3] = lop3_splice(w8, 0x00F000F0u, 0x64806480u);
}

// 4 int8 codes -> FP16 pairs (e0,e1), (e2,e3) holding 1152 + q.  Exact.
__device__ __forceinline__ void dequant_q8_biased(uint32_t w, uint32_t &p01, uint32_t &p23) {
  const uint32_t u = w ^ 0x80808080u;
  p01 = __byte_perm(u, 0x64646464u, 0x4140);
  p23 = __byte_perm(u, 0x64646464u, 0x4342);
}

// --------------------------------------------------------------- dec_main --
template <int B, int NT>
__global__ void __launch_bounds__(kDecThreads, 1) dec_main_kernel(
    const __grid_constant__ CUtensorMap mq4, const __grid_constant__ CUtensorMap ms4,
    const __grid_constant__ CUtensorMap mq8, const __grid_constant__ CUtensorMap mv,
    const __grid_constant__ CUtensorMap mq4q, const __grid_constant__ CUtensorMap ms4q,
    DecodeParams p) {
  constexpr int NTOK = 8 * NT;
  constexpr int P = B / 16;                 // threads per Hadamard block-row
  constexpr int NBLK = kSlab / B;           // Hadamard blocks per slab
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *q4s = base + p.L.q4;
  uint16_t *s4s = reinterpret_cast<uint16_t *>(base + p.L.s4);
  uint8_t *q8s = base + p.L.q8;
  __half *xq = reinterpret_cast<__half *>(base + p.L.xq);     // [ns][NTOK][kXRow]
  __half *xs = reinterpret_cast<__half *>(base + p.L.xs);     // [ns][NTOK][kXsRow]
  float *corr = reinterpret_cast<float *>(base + p.L.corr);   // [ns][4][NTOK]
  float *c8 = reinterpret_cast<float *>(base + p.L.c8);       // [ns][NBLK][NTOK]
  float *s8s = reinterpret_cast<float *>(base + p.L.s8);      // [upc][16]
  int16_t *colpos = reinterpret_cast<int16_t *>(base + p.L.colpos);   // [ns][256]
  int *samp = reinterpret_cast<int *>(base + p.L.samp);       // [kSamples]
  float *scr = reinterpret_cast<float *>(base + p.L.scr);
  int *meta = reinterpret_cast<int *>(base + p.L.meta);
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + p.L.bars);   // [upc_max + 2]
  uint16_t *vs = reinterpret_cast<uint16_t *>(base + p.L.vs);       // [rank][kSlab] BF16
  int *lo = meta;                                   // [kDecMaxSlabs + 1]
  int *lo16 = meta + 8;                             // [kDecMaxSlabs]
  int *nch = meta + 16;                             // [kDecMaxSlabs]
  int *q8off = meta + 24;                           // [kDecMaxUnits]
  int *flags = meta + 24 + kDecMaxUnits;            // [0]: the INT8 layout is valid

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int u0 = (int)(((long long)blockIdx.x * p.units) / p.grid);
  const int u1 = (int)(((long long)(blockIdx.x + 1) * p.units) / p.grid);
  const int nu = u1 - u0;
  if (nu <= 0) {
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  const int s_first = u0 / p.ntile;
  const int ns = (u1 - 1) / p.ntile - s_first + 1;
  if (ns > p.ns_max || nu > p.upc_max) {           // the host plan rules this out
    if (tid == 0) set_error(kErrBadShape);
    pdl_wait();
    pdl_launch_dependents();
    return;
  }

  // the first slab whose t share this CTA writes (the CTA holding its first unit)
  int own_si = -1;
  for (int si = 0; si < ns; ++si)
    if ((s_first + si) * p.ntile >= u0) { own_si = si; break; }
  uint64_t *q8bar = bars + p.upc_max;       // consumers -> producer: the INT8 layout is ready
  uint64_t *vbar = bars + p.upc_max + 1;    // V rows of the owned slab have landed

  // ------------- before the dependency wait: packed weights only -------------
  // Warp 0 is the producer: it initialises the barriers, issues the V rows
  // of the owned slab and every weight box, waits for the consumers' INT8
  // layout and issues the INT8 chunks, then leaves.  An issue can block while
  // the copy queue is full; the consumers (warps 1..15, named barrier 1)
  // never wait behind it.
  if (warp == 0) {
    for (int k = lane; k < nu; k += 32) mbar_init(&bars[k], 2);
    if (lane == 0) {
      mbar_init(q8bar, 1);
      mbar_init(vbar, 1);
    }
    fence_mbarrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&mq4);
      if (own_si >= 0 && p.rank > 0) {
        mbar_arrive_expect_tx(vbar, (uint32_t)(p.rank * kSlab * 2));
        tma_load_2d(vs, &mv, kSlab * (s_first + own_si), 0, vbar);
      } else {
        mbar_arrive(vbar);
      }
    }
    __syncwarp();
    const uint32_t bytes = kQ4Unit + (p.s4_tma ? kS4Unit : 0);
    for (int k = lane; k < nu; k += 32) {
      const int u = u0 + k, s = u / p.ntile, tile = u - s * p.ntile;
      const int lead = quad_lead(u, u0, u1, p.ntile, p.quad);
      if (lead == k) {
        mbar_arrive_expect_tx(&bars[k], 4 * bytes);
        tma_load_2d(q4s + k * kQ4Unit, &mq4q, s * 128, tile * kUnitRows, &bars[k]);
        if (p.s4_tma)
          tma_load_2d(s4s + k * (kS4Unit / 2), &ms4q, 8 * (s >> 1), tile * kUnitRows, &bars[k]);
      } else if (lead >= 0) {
        mbar_arrive(&bars[k]);          // its data comes with the quad's first unit
      } else {
        mbar_arrive_expect_tx(&bars[k], bytes);
        tma_load_2d(q4s + k * kQ4Unit, &mq4, s * 128, tile * kUnitRows, &bars[k]);
        if (p.s4_tma)
          tma_load_2d(s4s + k * (kS4Unit / 2), &ms4, 8 * (s >> 1), tile * kUnitRows, &bars[k]);
      }
    }
    // INT8 chunks: a unit's chunks are staged by TMA when they fit in the
    // budget (units in order), read from global memory otherwise
    const bool ready = mbar_wait(q8bar, 0);
    for (int k = lane; k < nu; k += 32) {
      const int u = u0 + k, s = u / p.ntile, tile = u - s * p.ntile, si = s - s_first;
      const int n = (ready && q8off[k] + nch[si] * kQ8Chunk <= p.q8_budget) ? nch[si] : 0;
      mbar_arrive_expect_tx(&bars[k], (uint32_t)(n * kQ8Chunk));
      for (int c = 0; c < n; ++c)
        tma_load_2d(q8s + q8off[k] + c * kQ8Chunk, &mq8, lo16[si] + 16 * c, tile * kUnitRows,
                    &bars[k]);
    }
    return;
  }
  const int ctid = tid - 32, cw = warp - 1;
  const int KG = p.K / 64;
  const int step = (p.n_sal + kSamples - 1) / kSamples;
  if (p.n_sal > 0)
    for (int i = ctid; i < kSamples; i += kDecConsThreads)
      samp[i] = __ldg(p.sal_idx + min(i * step, p.n_sal - 1));
  for (int i = ctid; i < nu * kUnitRows; i += kDecConsThreads) {
    const int k = i >> 4, r = i & 15;
    const int u = u0 + k, s = u / p.ntile, tile = u - s * p.ntile;
    const int m = tile * kUnitRows + r;
    s8s[i] = (m < p.M && p.n_sal > 0) ? bf16_bits_to_f32(p.s8[m]) : 0.0f;
  }
  if (!p.s4_tma) {
    // scale rows whose stride a tensor map cannot carry: plain loads
    for (int i = ctid; i < nu * kUnitRows * 8; i += kDecConsThreads) {
      const int k = i >> 7, r = (i >> 3) & 15, j = i & 7;
      const int u = u0 + k, s = u / p.ntile, tile = u - s * p.ntile;
      const int m = tile * kUnitRows + r, gcol = 8 * (s >> 1) + j;
      s4s[i] = (m < p.M && gcol < KG) ? p.s4[(size_t)m * KG + gcol] : (uint16_t)0;
    }
  }
  for (int i = ctid; i < ns * kSlab; i += kDecConsThreads) colpos[i] = -1;
  for (int i = ctid; i < ns * NTOK * kXsRow / 2; i += kDecConsThreads)
    reinterpret_cast<uint32_t *>(xs)[i] = 0u;
  // rows of V for further owned slabs (rare): warm L2
  if (p.rank > 0)
    for (int si = own_si + 1; own_si >= 0 && si < ns; ++si) {
      const int s = s_first + si;
      if (s * p.ntile < u0) continue;
      for (int i = ctid; i < p.rank * 4; i += kDecConsThreads) {
        const int rr = i >> 2, col = kSlab * s + 64 * (i & 3);
        if (col < p.K)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(p.V + (size_t)rr * p.K + col));
      }
    }
  dec_consumer_sync();

  // salient entries of each slab: lo[b] = #{e : sal_idx[e] < 256 (s_first + b)}
  if (cw <= ns) {
    int l = 0;
    if (p.n_sal > 0) {
      const int v = kSlab * (s_first + cw);
      int j = 0;
      for (int i0 = 0; i0 < kSamples; i0 += 32) {
        const int i = i0 + lane;
        j += __popc(__ballot_sync(0xffffffffu, i * step < p.n_sal && samp[i] < v));
      }
      // entries below v: all of [0, (j-1) step] plus some of ((j-1) step, j step)
      const int lb = j > 0 ? (j - 1) * step + 1 : 0;
      const int le = min(j * step, p.n_sal);
      int cnt = 0;
      for (int e = lb + lane; e < le; e += 32) cnt += __ldg(p.sal_idx + e) < v;
#pragma unroll
      for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      l = lb + cnt;
    }
    if (lane == 0) lo[cw] = l;
  }
  dec_consumer_sync();
  if (ctid < ns) {
    const int a = lo[ctid], b = lo[ctid + 1];
    lo16[ctid] = a & ~15;
    nch[ctid] = b > a ? (b - (a & ~15) + 15) >> 4 : 0;
  }
  dec_consumer_sync();
  if (cw == 0) {
    // q8 staging offsets: exclusive scan of the units' chunk bytes, then the
    // producer may issue the chunks (the arrive releases these writes)
    int run = 0;
    for (int k0 = 0; k0 < nu; k0 += 32) {
      const int k = k0 + lane;
      const int b = k < nu ? nch[(u0 + k) / p.ntile - s_first] * kQ8Chunk : 0;
      int inc = b;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
      }
      if (k < nu) q8off[k] = run + inc - b;
      run += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) flags[0] = 1;
    __syncwarp();
    if (lane == 0) mbar_arrive(q8bar);
  } else {
    // column -> position of each salient entry in its slab's chunk range
    for (int si = 0; si < ns; ++si) {
      const int a = lo[si], b = lo[si + 1], s = s_first + si;
      for (int e = a + ctid - 32; e < b; e += kDecConsThreads - 32) {
        const int col = __ldg(p.sal_idx + e) - kSlab * s;
        if (col >= 0 && col < kSlab) colpos[si * kSlab + col] = (int16_t)(e - (a & ~15));
      }
    }
  }
  dec_consumer_sync();

  // ------------------------- after the wait: activations -------------------------
  pdl_wait();
  pdl_launch_dependents();

  // rotate x for the CTA's slabs: block-row br = (si * NBLK + blk) * T + tok
  {
    const int nbr = ns * NBLK * p.T;
    const int grp = ctid / P, t = ctid % P;
    const int wgrp = (cw * 32) / P;              // first group of this warp
    for (int br0 = 0; br0 < nbr; br0 += p.nscr) {
      if (wgrp >= p.nscr || br0 + wgrp >= nbr) continue;   // whole warp idle
      const int br = br0 + grp;
      const bool live = br < nbr;                  // grp < nscr: nscr is whole warps
      const int tok = live ? br % p.T : 0;
      const int blk = live ? (br / p.T) % NBLK : 0;
      const int si = live ? br / (p.T * NBLK) : 0;
      const int col0 = kSlab * (s_first + si) + B * blk;
      float v[16];
#pragma unroll
      for (int a = 0; a < 16; ++a) {
        const int col = col0 + P * a + t;
        v[a] = (live && col < p.K) ? bf16_bits_to_f32(p.x[(size_t)tok * p.K + col]) : 0.0f;
      }
      fwht_group<B>(v, scr + grp * GroupScratch<B>::kElems, t);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] *= p.c;
      const int cs = B * blk + 16 * t;            // slab column of v[0]
      uint32_t h[8];
      float se = 0.0f, so = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j0 = perm16(2 * i), j1 = perm16(2 * i + 1);
        const __half a0 = __float2half_rn((j0 & 1) ? v[j0] * 0.0625f : v[j0]);
        const __half a1 = __float2half_rn((j1 & 1) ? v[j1] * 0.0625f : v[j1]);
        h[i] = pack_half2(a0, a1);
        if (j0 & 1) so += __half2float(a0); else se += __half2float(a0);
        if (j1 & 1) so += __half2float(a1); else se += __half2float(a1);
      }
      // bias term of the 64-column group: its four threads are adjacent lanes
      float cp = 1032.0f * se + 1152.0f * so;
      cp += __shfl_xor_sync(0xffffffffu, cp, 1);
      cp += __shfl_xor_sync(0xffffffffu, cp, 2);
      if (live) {
        uint4 *dst = reinterpret_cast<uint4 *>(xq + (size_t)(si * NTOK + tok) * kXRow + cs);
        dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
        dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
        if ((t & 3) == 0) corr[(si * 4 + cs / 64) * NTOK + tok] = cp;
      }
      // salient bias term of the block: 1152 x the sum of its salient x, as
      // stored in FP16 (the group's threads are adjacent lanes)
      float sal = 0.0f;
      if (live) {
        const int16_t *cpos = colpos + si * kSlab + cs;
        __half *xrow = xs + (size_t)(si * NTOK + tok) * kXsRow;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int pos = cpos[j];
          if (pos >= 0) {
            const __half hv = __float2half_rn(v[j]);
            xrow[pos] = hv;
            sal += __half2float(hv);
          }
        }
      }
#pragma unroll
      for (int o = 1; o < P; o <<= 1) sal += __shfl_xor_sync(0xffffffffu, sal, o);
      if (live && t == 0) c8[(si * NBLK + blk) * NTOK + tok] = 1152.0f * sal;
    }
  }
  dec_consumer_sync();

  // t share of each owned slab: tpart[s][rr][tok] = sum_j V[rr][j] x_rot[j],
  // on the tensor cores against the FP16 x_rot already in shared memory:
  // A = V in the same column order, odd columns scaled by 16 (x_rot holds
  // them divided by 16).  Warps split the 16-rank tiles and the K steps;
  // their partials go to the rotation scratch (free now) and are added in
  // warp order.  The first owned slab's V rows came by TMA; a further one is
  // read from global memory.
  const bool v_ok = p.rank == 0 || mbar_wait(vbar, 0);
  if (p.rank > 0) {
    const int mtiles = (p.rank + 15) / 16;
    const int kgp = max(1, kDecCons / mtiles);       // warps per rank tile
    float *tps = scr;                                // [mtiles][kgp][16][NTOK]
    const int mt = cw / kgp, kg = cw - mt * kgp;
    for (int si = own_si; si >= 0 && si < ns; ++si) {
      const int s = s_first + si;
      if (s * p.ntile < u0) continue;
      if (mt < mtiles) {
        const bool staged_v = si == own_si && v_ok;
        float d[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.0f;
        for (int ks = kg; ks < kSlab / 16; ks += kgp) {
          const int k0 = 16 * ks;
          uint32_t a[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int rr = 16 * mt + g + 8 * (h & 1);
            const int pos = k0 + 2 * tig + 8 * (h >> 1);
            __half e[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int col = ((pos + q) & ~15) + perm16((pos + q) & 15);
              float v = 0.0f;
              if (rr < p.rank && kSlab * s + col < p.K)
                v = bf16_bits_to_f32(staged_v ? vs[rr * kSlab + col]
                                              : p.V[(size_t)rr * p.K + kSlab * s + col]);
              e[q] = __float2half_rn((col & 1) ? v * 16.0f : v);
            }
            a[h] = pack_half2(e[0], e[1]);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const __half *xrow = xq + (size_t)(si * NTOK + 8 * nt + g) * kXRow + k0 + 2 * tig;
            const uint32_t b0 = *reinterpret_cast<const uint32_t *>(xrow);
            const uint32_t b1 = *reinterpret_cast<const uint32_t *>(xrow + 8);
            mma_16816(d[nt], a, b0, b1, d[nt]);
          }
        }
        float *dst = tps + (size_t)(mt * kgp + kg) * 16 * NTOK;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[(g + 8 * (i >> 1)) * NTOK + 8 * nt + 2 * tig + (i & 1)] = d[nt][i];
      }
      dec_consumer_sync();
      for (int i = ctid; i < p.rank * p.T; i += kDecConsThreads) {
        const int rr = i / p.T, tok = i - rr * p.T, m16 = rr >> 4, r = rr & 15;
        float v = 0.0f;
        for (int j = 0; j < kgp; ++j) v += tps[((size_t)(m16 * kgp + j) * 16 + r) * NTOK + tok];
        p.tpart[((size_t)s * p.rank + rr) * p.T + tok] = v;
      }
      dec_consumer_sync();
    }
  }
  dec_consumer_sync();

  // ----------------------------------- units -----------------------------------
  (void)flags;
  uint32_t bq[NT == 1 ? 4 : 1][8];
  int cur = -1;
  for (int k = cw; k < nu; k += kDecCons) {
    const int u = u0 + k, s = u / p.ntile, tile = u - s * p.ntile, si = s - s_first;
    if constexpr (NT == 1) {
      if (si != cur) {
        const __half *xrow = xq + (size_t)(si * NTOK + g) * kXRow + 16 * tig;
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          const uint4 x0 = *reinterpret_cast<const uint4 *>(xrow + 64 * gi);
          const uint4 x1 = *reinterpret_cast<const uint4 *>(xrow + 64 * gi + 8);
          bq[gi][0] = x0.x; bq[gi][1] = x0.y; bq[gi][2] = x0.z; bq[gi][3] = x0.w;
          bq[gi][4] = x1.x; bq[gi][5] = x1.y; bq[gi][6] = x1.z; bq[gi][7] = x1.w;
        }
        cur = si;
      }
    }
    if (!mbar_wait(&bars[k], 0)) break;
    {
      const int lead = quad_lead(u, u0, u1, p.ntile, p.quad);
      if (lead >= 0 && lead != k && !mbar_wait(&bars[lead], 0)) break;
    }
    const uint8_t *bx = q4s + k * kQ4Unit;
    const uint16_t *sb = s4s + k * (kS4Unit / 2) + 4 * (s & 1);
    const uint2 sl = *reinterpret_cast<const uint2 *>(sb + g * 8);
    const uint2 sh = *reinterpret_cast<const uint2 *>(sb + (g + 8) * 8);
    const uint32_t slw[4] = {sl.x & 0xFFFFu, sl.x >> 16, sl.y & 0xFFFFu, sl.y >> 16};
    const uint32_t shw[4] = {sh.x & 0xFFFFu, sh.x >> 16, sh.y & 0xFFFFu, sh.y >> 16};
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;

#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      const int chunk = 2 * gi + (tig >> 1);
      const uint32_t off = (uint32_t)(((chunk ^ g) << 4) + 8 * (tig & 1));
      const uint2 wl = *reinterpret_cast<const uint2 *>(bx + g * 128 + off);
      const uint2 wh = *reinterpret_cast<const uint2 *>(bx + (g + 8) * 128 + off);
      uint32_t fl[8], fh[8];
      dequant_q4_biased(wl.x, fl);
      dequant_q4_biased(wl.y, fl + 4);
      dequant_q4_biased(wh.x, fh);
      dequant_q4_biased(wh.y, fh + 4);
      const float slo = bf16_bits_to_f32(slw[gi]), shi = bf16_bits_to_f32(shw[gi]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint32_t b[8];
        if constexpr (NT == 1) {
#pragma unroll
          for (int i = 0; i < 8; ++i) b[i] = bq[gi][i];
        } else {
          const __half *xrow =
              xq + (size_t)(si * NTOK + g + 8 * nt) * kXRow + 64 * gi + 16 * tig;
          const uint4 x0 = *reinterpret_cast<const uint4 *>(xrow);
          const uint4 x1 = *reinterpret_cast<const uint4 *>(xrow + 8);
          b[0] = x0.x; b[1] = x0.y; b[2] = x0.z; b[3] = x0.w;
          b[4] = x1.x; b[5] = x1.y; b[6] = x1.z; b[7] = x1.w;
        }
        const float2 cc =
            *reinterpret_cast<const float2 *>(corr + (si * 4 + gi) * NTOK + 8 * nt + 2 * tig);
        float d[4] = {-cc.x, -cc.y, -cc.x, -cc.y};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t a[4] = {fl[2 * q], fh[2 * q], fl[2 * q + 1], fh[2 * q + 1]};
          mma_16816(d, a, b[2 * q], b[2 * q + 1], d);
        }
        acc[nt][0] = fmaf(slo, d[0], acc[nt][0]);
        acc[nt][1] = fmaf(slo, d[1], acc[nt][1]);
        acc[nt][2] = fmaf(shi, d[2], acc[nt][2]);
        acc[nt][3] = fmaf(shi, d[3], acc[nt][3]);
      }
    }

    // salient INT8 chunks of this slab
    const int nc = nch[si];
    if (nc > 0) {
      float d8[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float2 cc = *reinterpret_cast<const float2 *>(c8 + si * NBLK * NTOK + 8 * nt + 2 * tig);
        if constexpr (NBLK == 2) {
          const float2 c2 = *reinterpret_cast<const float2 *>(c8 + (si * NBLK + 1) * NTOK + 8 * nt + 2 * tig);
          cc.x += c2.x;
          cc.y += c2.y;
        }
        d8[nt][0] = -cc.x; d8[nt][1] = -cc.y; d8[nt][2] = -cc.x; d8[nt][3] = -cc.y;
      }
      const int mlo = tile * kUnitRows + g;
      for (int c = 0; c < nc; ++c) {
        uint32_t wl = 0u, wh = 0u;
        if (q8off[k] + nc * kQ8Chunk <= p.q8_budget) {
          const uint8_t *cb = q8s + q8off[k] + c * kQ8Chunk;
          wl = *reinterpret_cast<const uint32_t *>(cb + g * 16 + 4 * tig);
          wh = *reinterpret_cast<const uint32_t *>(cb + (g + 8) * 16 + 4 * tig);
        } else {
          const size_t e = (size_t)lo16[si] + 16 * c + 4 * tig;
          if (mlo < p.M)
            wl = __ldg(reinterpret_cast<const uint32_t *>(p.q8 + (size_t)mlo * p.n_sal + e));
          if (mlo + 8 < p.M)
            wh = __ldg(reinterpret_cast<const uint32_t *>(p.q8 + (size_t)(mlo + 8) * p.n_sal + e));
        }
        uint32_t l01, l23, h01, h23;
        dequant_q8_biased(wl, l01, l23);
        dequant_q8_biased(wh, h01, h23);
        const uint32_t a[4] = {l01, h01, l23, h23};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint2 xv = *reinterpret_cast<const uint2 *>(
              xs + (size_t)(si * NTOK + g + 8 * nt) * kXsRow + 16 * c + 4 * tig);
          mma_16816(d8[nt], a, xv.x, xv.y, d8[nt]);
        }
      }
      const float s8lo = s8s[k * 16 + g], s8hi = s8s[k * 16 + g + 8];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[nt][0] = fmaf(s8lo, d8[nt][0], acc[nt][0]);
        acc[nt][1] = fmaf(s8lo, d8[nt][1], acc[nt][1]);
        acc[nt][2] = fmaf(s8hi, d8[nt][2], acc[nt][2]);
        acc[nt][3] = fmaf(s8hi, d8[nt][3], acc[nt][3]);
      }
    }

    // this unit's partial of slab s
    const int m = tile * kUnitRows + g;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tok = 8 * nt + 2 * tig;
      float *dst = p.part + ((size_t)s * p.T + tok) * p.M;
      if (tok < p.T) {
        if (m < p.M) dst[m] = acc[nt][0];
        if (m + 8 < p.M) dst[m + 8] = acc[nt][2];
      }
      if (tok + 1 < p.T) {
        if (m < p.M) dst[p.M + m] = acc[nt][1];
        if (m + 8 < p.M) dst[p.M + m + 8] = acc[nt][3];
      }
    }
  }
}

// --------------------------------------------------------------- dec_tail --
// CTA = 64 rows of one token; thread (q, r) sums the q-th quarter of the
// slabs for row r, and the quarters are added in order.
__global__ void __launch_bounds__(kTailThreads) dec_tail_kernel(DecodeParams p) {
  constexpr int R = kTailThreads / 4;
  __shared__ float ts[64];
  __shared__ float tq[4][64];
  __shared__ float pq[4][R];
  const int q = threadIdx.x / R, r = threadIdx.x % R;
  const int m = blockIdx.x * R + r, tok = blockIdx.y;
  const bool live = m < p.M;
  // packed inputs first: they are not produced upstream
  uint4 ur[2];
  ur[0] = ur[1] = make_uint4(0u, 0u, 0u, 0u);
  if (live)
    for (int i = 0; i < 2; ++i) {
      const int rr = 8 * (2 * q + i);
      if (rr < p.rank) ur[i] = *reinterpret_cast<const uint4 *>(p.U + (size_t)m * p.rank + rr);
    }
  const float bv = (live && p.bias && q == 0) ? bf16_bits_to_f32(p.bias[m]) : 0.0f;
  pdl_wait();
  pdl_launch_dependents();
  const int nsl = p.nslices;
  // t = V x_rot: slab quarter q of rank index r
  if (r < p.rank) {
    const int s0 = (q * p.nslab) / 4, s1 = ((q + 1) * p.nslab) / 4;
    float t = 0.0f;
    int s = s0;
    for (; s + 8 <= s1; s += 8) {
      float tv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) tv[i] = __ldcg(&p.tpart[((size_t)(s + i) * p.rank + r) * p.T + tok]);
#pragma unroll
      for (int i = 0; i < 8; ++i) t += tv[i];
    }
    for (; s < s1; ++s) t += __ldcg(&p.tpart[((size_t)s * p.rank + r) * p.T + tok]);
    tq[q][r] = t;
  }
  float v = 0.0f;
  if (live) {
    const int s0 = (q * nsl) / 4, s1 = ((q + 1) * nsl) / 4;
    const float *src = p.part + (size_t)tok * p.M + m;
    const size_t stride = (size_t)p.T * p.M;
    int s = s0;
    for (; s + 16 <= s1; s += 16) {
      float pv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) pv[i] = __ldcg(src + (size_t)(s + i) * stride);
#pragma unroll
      for (int i = 0; i < 16; ++i) v += pv[i];
    }
    float pv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) pv[i] = s + i < s1 ? __ldcg(src + (size_t)(s + i) * stride) : 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) v += pv[i];
  }
  pq[q][r] = v;
  __syncthreads();
  if (threadIdx.x < p.rank)
    ts[threadIdx.x] = ((tq[0][threadIdx.x] + tq[1][threadIdx.x]) + tq[2][threadIdx.x]) + tq[3][threadIdx.x];
  __syncthreads();
  // U t: quarter q takes rank indices [16q, 16q + 16)
  float ut = 0.0f;
  for (int i = 0; i < 2; ++i) {
    const int rr = 8 * (2 * q + i);
    if (rr >= p.rank) break;
    const uint32_t w[4] = {ur[i].x, ur[i].y, ur[i].z, ur[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ut = fmaf(bf16_bits_to_f32(w[j] & 0xFFFFu), ts[rr + 2 * j], ut);
      ut = fmaf(bf16_bits_to_f32(w[j] >> 16), ts[rr + 2 * j + 1], ut);
    }
  }
  __syncthreads();
  tq[q][r] = ut;
  __syncthreads();
  if (q != 0 || !live) return;
  float y = ((pq[0][r] + pq[1][r]) + pq[2][r]) + pq[3][r];
  y += ((tq[0][r] + tq[1][r]) + tq[2][r]) + tq[3][r];
  y += bv;
  if (p.y_bf16)
    reinterpret_cast<uint16_t *>(p.y)[(size_t)tok * p.M + m] = f32_to_bf16_rn_bits(y);
  else
    reinterpret_cast<float *>(p.y)[(size_t)tok * p.M + m] = y;
}

// ---------------------------------------------------------------- host ---
namespace {

std::mutex g_sm_mu;
std::vector<int> g_sm_count;

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lk(g_sm_mu);
  if ((int)g_sm_count.size() <= dev) g_sm_count.resize(dev + 1, 0);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

struct DecPlan {
  int nslab, ntile, units, grid, upc_max, ns_max, NT, ntok, nscr, q8_budget;
  DecLayout L;
  bool ok;
};

int slabs_spanned(long long units, int grid, int ntile, int c) {
  const int u0 = (int)((c * units) / grid), u1 = (int)(((c + 1) * units) / grid);
  if (u1 <= u0) return 0;
  return (u1 - 1) / ntile - u0 / ntile + 1;
}

// Grid, per-CTA maxima and the shared-memory layout of one decode call.
DecPlan dec_plan(int M, int K, int block, int T, int rank, int nsm) {
  DecPlan d{};
  d.nslab = (K + kSlab - 1) / kSlab;
  d.ntile = (M + kUnitRows - 1) / kUnitRows;
  d.units = d.nslab * d.ntile;
  d.NT = T <= 8 ? 1 : 2;
  d.ntok = 8 * d.NT;
  int grid = std::min(d.units, nsm);
  for (;;) {
    const int upc = (d.units + grid - 1) / grid;
    int ns = 0;
    for (int c = 0; c < grid; ++c) ns = std::max(ns, slabs_spanned(d.units, grid, d.ntile, c));
    if ((upc <= kDecMaxUnits && ns <= kDecMaxSlabs) || grid >= d.units) {
      d.grid = grid;
      d.upc_max = upc;
      d.ns_max = ns;
      break;
    }
    grid = std::min(d.units, grid + std::max(1, grid / 4));
  }
  const int P = block / 16;
  const int gpw = 32 / P;                          // Hadamard groups per warp
  const int nbr = d.ns_max * (kSlab / block) * T;
  int nscr = std::min(nbr, block == 256 ? 16 : 32);
  nscr = (nscr + gpw - 1) / gpw * gpw;             // whole warps
  d.nscr = nscr;
  const int scr_elems = 16 * (P + 1) + 1;
  auto al = [](int v, int a) { return (v + a - 1) / a * a; };
  DecLayout &L = d.L;
  int off = 0;
  L.q4 = off;     off += d.upc_max * kQ4Unit;
  L.s4 = off;     off += d.upc_max * kS4Unit;
  L.xq = off;     off += al(d.ns_max * d.ntok * kXRow * 2, 128);
  L.xs = off;     off += al(d.ns_max * d.ntok * kXsRow * 2, 128);
  L.corr = off;   off += al(d.ns_max * 4 * d.ntok * 4, 128);
  L.c8 = off;     off += al(d.ns_max * 2 * d.ntok * 4, 128);
  L.s8 = off;     off += al(d.upc_max * kUnitRows * 4, 128);
  L.colpos = off; off += al(d.ns_max * kSlab * 2, 128);
  L.samp = off;   off += kSamples * 4;
  // the rotation scratch also holds the t-share partials: at most 15 warps x
  // 16 ranks x the token tile, FP32
  L.scr = off;    off += al(std::max(d.nscr * scr_elems * 4, kDecCons * 16 * d.ntok * 4), 128);
  L.meta = off;   off += 512;
  L.bars = off;   off += al((d.upc_max + 2) * 8, 128);
  L.vs = off;     off += al(rank * kSlab * 2, 128);
  L.q8 = off;
  const int room = kSmemLimit - 1024 - off;
  d.q8_budget = std::max(0, std::min(room, d.upc_max * 17 * kQ8Chunk)) / kQ8Chunk * kQ8Chunk;
  off += d.q8_budget;
  L.total = off + 1024;
  d.ok = room >= 0 && d.upc_max <= kDecMaxUnits && d.ns_max <= kDecMaxSlabs;
  return d;
}

}  // namespace

size_t decode_row_slices(int K, int n_sal);

size_t decode_workspace_bytes(int M, int K, int block, int n_sal, int rank, int T) {
  (void)block;
  const size_t nslab = (size_t)(K + kSlab - 1) / kSlab;
  const size_t slices = T <= 2 ? std::max(nslab, decode_row_slices(K, n_sal)) : nslab;
  size_t off = 0;
  auto take = [&](size_t b) { off += (b + 255) & ~(size_t)255; };
  take(slices * T * M * 4);            // partials (per slab, or per CTA of a tile)
  take(nslab * rank * T * 4 + 16);     // per-slab shares of t = V x_rot
  return off;
}

cudaError_t launch_decode_row(const ForwardArgs &a, cudaStream_t st, Launcher &L);
cudaError_t prepare_decode_row_kernels();

cudaError_t launch_decode(const ForwardArgs &a, cudaStream_t st, Launcher &L) {
  if (a.T <= 2) {
    const cudaError_t e = launch_decode_row(a, st, L);
    if (e != cudaErrorNotSupported) return e;
  }
  const DecPlan d = dec_plan(a.M, a.K, a.block, a.T, a.rank, sm_count());
  if (!d.ok) {
    set_last_error("decode: no shared-memory plan fits this shape");
    return cudaErrorInvalidConfiguration;
  }
  DecodeParams p;
  p.M = a.M; p.K = a.K; p.T = a.T; p.n_sal = a.n_sal; p.rank = a.rank; p.block = a.block;
  p.nslab = d.nslab; p.ntile = d.ntile; p.units = d.units; p.grid = d.grid;
  p.upc_max = d.upc_max; p.ns_max = d.ns_max; p.ntok = d.ntok; p.nscr = d.nscr;
  p.q8_budget = d.q8_budget;
  p.c = (float)sqrt(1.0 / (double)a.block);
  p.s4 = a.s4; p.sal_idx = a.sal_idx; p.q8 = a.q8; p.s8 = a.s8; p.U = a.U; p.V = a.V;
  p.x = a.x; p.bias = a.bias; p.y = a.y; p.y_bf16 = a.y_bf16;
  p.L = d.L;
  p.nslices = d.nslab;
  char *ws = static_cast<char *>(a.workspace);
  size_t off = 0;
  auto take = [&](size_t b) { char *q = ws + off; off += (b + 255) & ~(size_t)255; return q; };
  p.part = reinterpret_cast<float *>(take((size_t)d.nslab * a.T * a.M * 4));
  p.tpart = reinterpret_cast<float *>(take((size_t)d.nslab * a.rank * a.T * 4 + 16));

  CUtensorMap mq4, ms4, mq8, mv;
  if (encode_tmap_2d(&mq4, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q4, (uint64_t)a.K / 2, (uint64_t)a.M,
                     (uint64_t)a.K / 2, 128, kUnitRows, CU_TENSOR_MAP_SWIZZLE_128B) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // s4 rows are K/32 bytes: a tensor map needs a multiple of 16
  p.s4_tma = (a.K % 512 == 0) && ((uintptr_t)a.s4 % 16 == 0);
  ms4 = mq4;
  if (p.s4_tma && encode_tmap_2d(&ms4, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.s4, (uint64_t)a.K / 64,
                                 (uint64_t)a.M, (uint64_t)a.K / 32, 8, kUnitRows,
                                 CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
    p.s4_tma = 0;
  // four tiles of one slab per box (the same bytes, a quarter of the copies)
  CUtensorMap mq4q = mq4, ms4q = mq4;
  p.quad = encode_tmap_2d(&mq4q, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q4, (uint64_t)a.K / 2,
                          (uint64_t)a.M, (uint64_t)a.K / 2, 128, 4 * kUnitRows,
                          CU_TENSOR_MAP_SWIZZLE_128B) == CUDA_SUCCESS &&
           (!p.s4_tma ||
            encode_tmap_2d(&ms4q, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.s4, (uint64_t)a.K / 64,
                           (uint64_t)a.M, (uint64_t)a.K / 32, 8, 4 * kUnitRows,
                           CU_TENSOR_MAP_SWIZZLE_NONE) == CUDA_SUCCESS);
  // V rows of one slab: box {256 columns, rank rows}
  mv = mq4;    // never read when rank == 0
  if (a.rank > 0 &&
      encode_tmap_2d(&mv, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.V, (uint64_t)a.K, (uint64_t)a.rank,
                     (uint64_t)a.K * 2, kSlab, (uint32_t)a.rank, CU_TENSOR_MAP_SWIZZLE_NONE) !=
          CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  mq8 = mq4;   // never read when there are no salient columns
  if (a.n_sal > 0 &&
      encode_tmap_2d(&mq8, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q8, (uint64_t)a.n_sal, (uint64_t)a.M,
                     (uint64_t)a.n_sal, 16, kUnitRows, CU_TENSOR_MAP_SWIZZLE_NONE) !=
          CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  cudaError_t e;
  const dim3 grid(d.grid), block(kDecThreads);
  const size_t smem = d.L.total;
  if (a.block == 256)
    e = d.NT == 1 ? L.launch("dec_main", dec_main_kernel<256, 1>, grid, block, smem, st, true,
                             mq4, ms4, mq8, mv, mq4q, ms4q, p)
                  : L.launch("dec_main", dec_main_kernel<256, 2>, grid, block, smem, st, true,
                             mq4, ms4, mq8, mv, mq4q, ms4q, p);
  else
    e = d.NT == 1 ? L.launch("dec_main", dec_main_kernel<128, 1>, grid, block, smem, st, true,
                             mq4, ms4, mq8, mv, mq4q, ms4q, p)
                  : L.launch("dec_main", dec_main_kernel<128, 2>, grid, block, smem, st, true,
                             mq4, ms4, mq8, mv, mq4q, ms4q, p);
  if (e != cudaSuccess) return e;
  return L.launch("dec_tail", dec_tail_kernel, dim3((a.M + kTailThreads / 4 - 1) / (kTailThreads / 4), a.T),
                  dim3(kTailThreads), 0, st, true, p);
}

cudaError_t prepare_decode_kernels() {
  cudaError_t e;
  for (const void *f :
       {(const void *)dec_main_kernel<256, 1>, (const void *)dec_main_kernel<256, 2>,
        (const void *)dec_main_kernel<128, 1>, (const void *)dec_main_kernel<128, 2>}) {
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kSmemLimit)) != cudaSuccess)
      return e;
  }
  (void)sm_count();
  return prepare_decode_row_kernels();
}

}  // namespace dvssq
