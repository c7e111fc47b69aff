// Decode-shaped forward for one or two tokens: the DV-SSQ runtime equation
// (MiniCPM5-2B-Hadamard-GSQ card, §2, Y = X What^T + (X B^T) A^T, with the
// Spark card's INT8 salient tier) as exact integer dot products on the CUDA
// cores.
//
// With so few tokens the layer is a pure weight stream: every weight is
// used T times.  Warp-level MMA would waste 7/8 of its N dimension, so this
// path keeps the contraction in 32-bit integers instead:
//   * the rotated activations x_rot = H x are held as int16 with one FP32
//     scale per 64-column group (|x| <= 32767 * scale, relative step 2^-15);
//   * an even column's nibble becomes the byte u = q + 8 in [0, 15] (one
//     LOP3 per four nibbles); an odd column's nibble, masked in place, is a
//     signed byte equal to 16 q (one AND per four); DP2A multiplies two int16
//     activations by two bytes;
//   * a 64-column group sum is exact in int32: the even-column sum minus
//     8 * (sum of the group's even-column int16 activations), plus the
//     odd-column sum divided by 16 (exactly), is sum q * x_int, and the group
//     result s4 * scale * sum is accumulated in FP32.
// The salient INT8 columns run the same way (signed bytes, no bias), with
// the salient activations requantised per 128-entry chunk.
//
// Work units are 2 KB: 16 rows x one 256-column slab of q4, or 16 rows x
// 128 salient entries of q8.  q4 units are numbered by column group (S
// slabs), then 16-row tile, then slab; the q8 units follow, by chunk then
// tile.  Each CTA (one per SM) takes an equal contiguous share, so it meets
// one or two column groups and a salient chunk or two: it rotates only the
// Hadamard blocks those cover, and every weight load is issued by TMA before
// the dependency wait.  Each (column group, tile) is split between at most
// two CTAs, which write partial slots 2g and 2g + 1 (the first writes a zero
// into the second when it holds the whole segment); each salient chunk has
// slot 2 * groups + chunk.  dec_tail sums a row's slots in order and adds
// U t + bias.

namespace dvssq {

constexpr int kRowWarps = 16;
constexpr int kRowThreads = 32 * kRowWarps;
constexpr int kRowMaxUnits = 64;
constexpr int kRowUnit = 2048;            // bytes of one unit (16 rows x 128 B)
constexpr int kRowSlots = 5;              // segments one warp's unit range can touch
constexpr int kCons = kRowWarps - 1;      // consumer warps (warp 0 issues the weight stream)
constexpr int kConsThreads = 32 * kCons;
constexpr int kRowGroupSlabs = 4;         // slabs per column group
constexpr int kRowMaxSlabMask = 8;        // 32-bit words of the slab mask (K <= 65536)

// Barrier among the consumer warps only: the producer warp may still be
// blocked issuing copies (or gone) when they synchronise.
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsThreads) : "memory");
}

struct RowLayout {
  int units, s4, x, xsc, xsum, xs, xss, sidx, s8, red, wt, scr, slist, vs, bars, total;
};

// Unit geometry of the column-group order.
struct RowGeom {
  int ntile, nslab, S, ng, Slast, nq4, nq8u;
};

struct RowUnit {
  int q8;     // 1 for a salient unit
  int g;      // column group (q4) or salient chunk (q8)
  int t;      // 16-row tile
  int j;      // slab (q4) or chunk (q8)
  int key;    // segment key: (group, tile) or (chunk, tile), increasing with u
};

// (Unit counts stay far below 2^31: the host plan caps the layer size.)
__host__ __device__ inline RowUnit row_unit(int u, const RowGeom &G) {
  RowUnit r;
  if (u < G.nq4) {
    const int full = (G.ng - 1) * G.ntile * G.S;
    int loc, Sg;
    if (u < full) {
      r.g = u / (G.ntile * G.S);
      loc = u - r.g * G.ntile * G.S;
      Sg = G.S;
    } else {
      r.g = G.ng - 1;
      loc = u - full;
      Sg = G.Slast;
    }
    r.q8 = 0;
    r.t = loc / Sg;
    r.j = r.g * G.S + (loc - r.t * Sg);
    r.key = r.g * G.ntile + r.t;
  } else {
    const int v = u - G.nq4;
    r.q8 = 1;
    r.g = r.j = v / G.ntile;
    r.t = v - r.g * G.ntile;
    r.key = G.ng * G.ntile + v;
  }
  return r;
}

// The unit after `r` in the column-group order.
__device__ __forceinline__ void row_unit_next(RowUnit &r, const RowGeom &G) {
  if (!r.q8) {
    const int Sg = r.g < G.ng - 1 ? G.S : G.Slast;
    if (++r.j < r.g * G.S + Sg) return;
    if (++r.t < G.ntile) { r.j = r.g * G.S; ++r.key; return; }
    r.t = 0;
    ++r.key;
    if (++r.g < G.ng) { r.j = r.g * G.S; return; }
    r.q8 = 1;
    r.g = r.j = 0;
    return;
  }
  ++r.key;
  if (++r.t < G.ntile) return;
  r.t = 0;
  ++r.g;
  ++r.j;
}

// First unit of the q4 segment (group g, tile t) and its slab count.
__host__ __device__ inline int seg_first(int g, int t, const RowGeom &G, int *Sg) {
  *Sg = g < G.ng - 1 ? G.S : G.Slast;
  return g * G.ntile * G.S + t * (*Sg);
}

// The unit that makes its CTA compute slab s's share of t: slab s at a
// tile spread over the group, so that a group's shares fall on different CTAs.
__host__ __device__ inline int t_owner_unit(int s, const RowGeom &G) {
  const int g = s / G.S, i = s - g * G.S;
  int Sg;
  const int first = seg_first(g, (i * G.ntile) / (g < G.ng - 1 ? G.S : G.Slast), G, &Sg);
  return first + i;
}

struct RowParams {
  int M, K, T, n_sal, rank, block;
  RowGeom G;
  int units, grid, upc_max, maxq8, nscr;
  int s4_tma;
  int QW;           // salient entries per q8 unit: 128, or n_sal when smaller
  float c;
  const uint16_t *s4;
  const int32_t *sal_idx;
  const uint16_t *s8;
  const uint16_t *V;
  const uint16_t *x;
  float *part;    // [slot][T][M]
  float *tpart;   // [nslab][rank][T]
  RowLayout L;
};

__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c) {
  return __dp2a_lo((int)a, (int)b, c);
}
__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c) {
  return __dp2a_hi((int)a, (int)b, c);
}

// Position of column j (0..7) of an 8-column segment in the DP2A order
// {0, 2, 4, 6, 1, 3, 5, 7} of the stored int16 activations.
__host__ __device__ constexpr int seg_pos(int j) { return (j & 1) ? 4 + (j >> 1) : (j >> 1); }

template <int B, int T>
__global__ void __launch_bounds__(kRowThreads, 1) dec_row_kernel(
    const __grid_constant__ CUtensorMap mq4, const __grid_constant__ CUtensorMap ms4,
    const __grid_constant__ CUtensorMap mq8, const __grid_constant__ CUtensorMap ms8,
    const __grid_constant__ CUtensorMap mv, RowParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *us = base + p.L.units;                                        // [upc][2048]
  uint16_t *s4s = reinterpret_cast<uint16_t *>(base + p.L.s4);           // [upc][16][8]
  int16_t *xi = reinterpret_cast<int16_t *>(base + p.L.x);               // [T][K]
  float *xsc = reinterpret_cast<float *>(base + p.L.xsc);                // [T][K/64]
  int *xsum = reinterpret_cast<int *>(base + p.L.xsum);                  // [T][K/64]
  int16_t *xs = reinterpret_cast<int16_t *>(base + p.L.xs);              // [chunk][T][128]
  float *xss = reinterpret_cast<float *>(base + p.L.xss);                // [chunk][T]
  int *sidx = reinterpret_cast<int *>(base + p.L.sidx);                  // [chunk][128]
  uint16_t *s8s = reinterpret_cast<uint16_t *>(base + p.L.s8);           // [q8 slot][64] BF16 (16 used)
  float *red = reinterpret_cast<float *>(base + p.L.red);                // [warp][seg][T][16]
  int *wt = reinterpret_cast<int *>(base + p.L.wt);                      // [warp][2]
  float *scr = reinterpret_cast<float *>(base + p.L.scr);                // FWHT transposes
  uint32_t *smask = reinterpret_cast<uint32_t *>(base + p.L.slist);      // [kRowMaxSlabMask]
  int *slist = reinterpret_cast<int *>(base + p.L.slist) + kRowMaxSlabMask + 1;   // [nslab]
  uint16_t *vs = reinterpret_cast<uint16_t *>(base + p.L.vs);           // [rank][256] BF16
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + p.L.bars);        // [upc] + x, s, v
  const RowGeom &G = p.G;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KG = p.K / 64;
  const int u0 = (int)(((long long)blockIdx.x * p.units) / p.grid);
  const int u1 = (int)(((long long)(blockIdx.x + 1) * p.units) / p.grid);
  const int nu = u1 - u0;
  if (nu <= 0 || nu > p.upc_max) {
    if (nu > p.upc_max && tid == 0) set_error(kErrBadShape);
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  const int q8first = max(u0, G.nq4);           // first salient unit (if any)
  const int nq8 = max(0, u1 - q8first);
  // salient chunks met by this CTA: the indices and activations are per chunk
  const int jj0 = nq8 > 0 ? (q8first - G.nq4) / G.ntile : 0;
  const int nchunk = nq8 > 0 ? (u1 - 1 - G.nq4) / G.ntile - jj0 + 1 : 0;
  uint64_t *xbar = &bars[p.upc_max];
  uint64_t *sbar = &bars[p.upc_max + 1];        // the salient indices of all q8 units
  uint64_t *vbar = &bars[p.upc_max + 2];        // V rows of the first owned t share
  // column groups of this CTA and the first slab whose t share it computes
  const int uq4_last = min(u1, G.nq4) - 1;
  const int gA = u0 < G.nq4 ? row_unit(u0, G).g : 0;
  const int gB = u0 < G.nq4 ? row_unit(uq4_last, G).g : -1;
  int s_own = -1;
  for (int g = gA; g <= gB && p.rank > 0 && s_own < 0; ++g)
    for (int s = g * G.S; s < min((g + 1) * G.S, G.nslab); ++s) {
      const int uf = t_owner_unit(s, G);
      if (uf >= u0 && uf < u1) { s_own = s; break; }
    }

  // ------------- before the dependency wait: packed weights only -------------
  // warp 0 sets up the barriers and then only issues the weight stream: an
  // issue blocks while the copy queue is full, so that warp does nothing
  // else; warps 1..15 do the rest.
  if (warp == 0) {
    for (int k = lane; k <= nu + 2; k += 32)
      mbar_init(k < nu ? &bars[k] : k == nu ? xbar : k == nu + 1 ? sbar : vbar, 1);
    fence_mbarrier_init();
  }
  if (tid < kRowMaxSlabMask) smask[tid] = 0u;
  __syncthreads();
  if (warp == 0) {
    // the salient indices first (small, needed before the rotation), then
    // the salient units, then the q4 units
    if (lane == 0) {
      if (s_own >= 0) {
        mbar_arrive_expect_tx(vbar, (uint32_t)(p.rank * kSlab * 2));
        tma_load_2d(vs, &mv, kSlab * s_own, 0, vbar);
      }
      uint32_t bytes = 0;
      for (int c = 0; c < nchunk; ++c) bytes += 4 * min(p.QW, p.n_sal - p.QW * (jj0 + c));
      mbar_arrive_expect_tx(sbar, bytes);
      for (int c = 0; c < nchunk; ++c) {
        const int jj = jj0 + c;
        bulk_g2s(sidx + c * 128, p.sal_idx + p.QW * jj, 4 * min(p.QW, p.n_sal - p.QW * jj), sbar);
      }
    }
    __syncwarp();
    for (int pass = 0; pass < 2; ++pass)
      for (int k = lane; k < nu; k += 32) {
        const int u = u0 + k;
        const RowUnit ru = row_unit(u, G);
        if (ru.q8 != (pass == 0)) continue;
        if (!ru.q8) {
          mbar_arrive_expect_tx(&bars[k], kRowUnit + (p.s4_tma ? 256 : 0));
          tma_load_2d(us + k * kRowUnit, &mq4, ru.j * 128, ru.t * 16, &bars[k]);
          if (p.s4_tma)
            tma_load_2d(s4s + k * 128, &ms4, 8 * (ru.j >> 1), ru.t * 16, &bars[k]);
        } else {
          const int slot = u - q8first;
          mbar_arrive_expect_tx(&bars[k], 16 * p.QW + 32);
          tma_load_2d(us + k * kRowUnit, &mq8, ru.j * p.QW, ru.t * 16, &bars[k]);
          tma_load_2d(s8s + slot * 64, &ms8, ru.t * 16, 0, &bars[k]);
        }
      }
    return;
  }
  const int cw = warp - 1, ctid = tid - 32;
  if (!p.s4_tma) {
    // scale rows whose stride a tensor map cannot carry: plain loads
    for (int i = ctid; i < nu * 128; i += kConsThreads) {
      const int k = i >> 7, r = (i >> 3) & 15, g = i & 7;
      const RowUnit ru = row_unit(u0 + k, G);
      const int m = ru.t * 16 + r, gcol = 8 * (ru.j >> 1) + g;
      if (!ru.q8)
        s4s[i] = (m < p.M && gcol < KG) ? p.s4[(size_t)m * KG + gcol] : (uint16_t)0;
    }
  }

  // ------------------------- after the wait: activations -------------------------
  pdl_wait();
  pdl_launch_dependents();
  if (ctid == 0) {
    mbar_arrive_expect_tx(xbar, (uint32_t)(T * p.K * 2));
    for (int tok = 0; tok < T; ++tok)
      bulk_g2s(xi + (size_t)tok * p.K, p.x + (size_t)tok * p.K, p.K * 2, xbar);
  }
  // slabs to rotate: the q4 column groups, and the slabs the salient chunks'
  // columns fall in (sal_idx is ascending, so a chunk spans first..last)
  for (int s = gA * G.S + ctid; gA <= gB && s < min((gB + 1) * G.S, G.nslab); s += kConsThreads)
    atomicOr(&smask[s >> 5], 1u << (s & 31));
  const bool s_ok = nq8 == 0 || mbar_wait(sbar, 0);
  for (int c = cw; c < nchunk && s_ok; c += kCons) {
    const int jj = jj0 + c;
    const int ne = min(p.QW, p.n_sal - p.QW * jj);
    const int c0 = sidx[c * 128], c1 = sidx[c * 128 + ne - 1];
    if (c0 < 0 || c1 >= p.K || c1 < c0) continue;          // sal_idx must be ascending
    for (int s = c0 / kSlab + lane; s <= c1 / kSlab; s += 32) atomicOr(&smask[s >> 5], 1u << (s & 31));
  }
  constexpr int NV = (64 + kCons - 1) / kCons;     // rank rows per consumer warp
  consumer_sync();                       // xbar armed, slab mask complete
  if (cw == 0) {
    int n = 0;
    for (int w = 0; w < kRowMaxSlabMask; ++w) {
      const uint32_t bits = smask[w];
      if (lane < 32 && (bits >> lane) & 1u) slist[n + __popc(bits & ((1u << lane) - 1u))] = 32 * w + lane;
      n += __popc(bits);
    }
    if (lane == 0) slist[-1] = n;
  }
  consumer_sync();
  const int nsl = slist[-1];
  const bool x_ok = mbar_wait(xbar, 0);

  // rotate the listed slabs of x in place: BF16 in, int16 (DP2A order) and a
  // per-group scale out.  A Hadamard block-row is P = B/16 threads
  // (16-thread Kronecker FWHT with a padded shared-memory transpose); thread
  // t ends with columns 16t..16t+15.
  {
    constexpr int P = B / 16, NBLK = kSlab / B;
    const int nbr = nsl * NBLK * T;
    const int grp = ctid / P, t = ctid % P;
    for (int br0 = 0; br0 < nbr && x_ok; br0 += p.nscr) {
      if ((cw * 32) / P >= p.nscr || br0 + (cw * 32) / P >= nbr) continue;   // whole warp idle
      const int br = br0 + grp;
      const bool live = grp < p.nscr && br < nbr;
      const int tok = live ? br % T : 0;
      const int kb = live ? slist[br / (NBLK * T)] * NBLK + (br / T) % NBLK : 0;
      uint16_t *blk = reinterpret_cast<uint16_t *>(xi) + (size_t)tok * p.K + kb * B;
      const bool in_k = live && kb * B < p.K;
      float v[16];
#pragma unroll
      for (int a = 0; a < 16; ++a) v[a] = in_k ? bf16_bits_to_f32(blk[P * a + t]) : 0.0f;
      fwht_group<B>(v, scr + (grp < p.nscr ? grp : 0) * GroupScratch<B>::kElems, t);
      float mx = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[j] *= p.c;
        mx = fmaxf(mx, fabsf(v[j]));
      }
      // a 64-column group is 4 adjacent threads
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float inv = mx > 0.0f ? 32767.0f / mx : 0.0f;
      int q[16], sum = 0;      // sum over the even columns (their codes carry the +8)
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        q[j] = max(-32767, min(32767, __float2int_rn(v[j] * inv)));
        if (!(j & 1)) sum += q[j];
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      if (in_k) {
        // the whole group has read its inputs (fwht_group synchronised the warp)
        uint4 w[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int *qq = q + 8 * hh;
          w[hh].x = (uint32_t)(qq[0] & 0xFFFF) | ((uint32_t)qq[2] << 16);
          w[hh].y = (uint32_t)(qq[4] & 0xFFFF) | ((uint32_t)qq[6] << 16);
          w[hh].z = (uint32_t)(qq[1] & 0xFFFF) | ((uint32_t)qq[3] << 16);
          w[hh].w = (uint32_t)(qq[5] & 0xFFFF) | ((uint32_t)qq[7] << 16);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(blk + 16 * t);
        dst[0] = w[0];
        dst[1] = w[1];
        if ((t & 3) == 0) {
          const int gcol = (kb * B + 16 * t) / 64;
          xsc[tok * KG + gcol] = mx * (1.0f / 32767.0f);
          xsum[tok * KG + gcol] = sum;
        }
      }
    }
  }
  consumer_sync();

  // salient activations of the CTA's chunks, requantised per chunk
  for (int w = cw; w < nchunk * T && s_ok; w += kCons) {
    const int slot = w / T, tok = w % T;      // slot = chunk - jj0
    const int jj = jj0 + slot;
    float val[4];
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = 4 * lane + i;
      val[i] = 0.0f;
      if (e < p.QW && p.QW * jj + e < p.n_sal) {
        const int col = sidx[slot * 128 + e];
        if (col >= 0 && col < p.K) {
          const int pos = (col & ~7) + seg_pos(col & 7);
          val[i] = (float)xi[(size_t)tok * p.K + pos] * xsc[tok * KG + col / 64];
        }
      }
      mx = fmaxf(mx, fabsf(val[i]));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float inv = mx > 0.0f ? 32767.0f / mx : 0.0f;
    int qv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) qv[i] = max(-32767, min(32767, __float2int_rn(val[i] * inv)));
    uint2 pk;
    pk.x = (uint32_t)(qv[0] & 0xFFFF) | ((uint32_t)qv[1] << 16);
    pk.y = (uint32_t)(qv[2] & 0xFFFF) | ((uint32_t)qv[3] << 16);
    *reinterpret_cast<uint2 *>(xs + ((size_t)slot * T + tok) * 128 + 4 * lane) = pk;
    if (lane == 0) xss[slot * T + tok] = mx * (1.0f / 32767.0f);
  }

  consumer_sync();      // x_rot and the salient activations are complete

  // t shares of the slabs this CTA owns (t_owner_unit), read only by the
  // tail kernel: no barrier follows.  Rank row rr goes to warp
  // kCons - 1 - rr % kCons, whose units are issued last and arrive last.
  // tpart[s][rr][tok] = sum over the slab of V[rr][j] x_rot[j]
  for (int g = gA; g <= gB && p.rank > 0; ++g)
    for (int s = g * G.S; s < min((g + 1) * G.S, G.nslab); ++s) {
      const int uf = t_owner_unit(s, G);
      if (uf < u0 || uf >= u1) continue;
      uint4 vreg[NV];
      const int c0 = kSlab * s + 8 * lane;          // 8 columns = one DP2A segment
      // the first owned slab came by TMA with the weights; a further one
      // (only for very wide layers) is read from global memory
      const bool staged = s == s_own && mbar_wait(vbar, 0);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int rr = (kCons - 1 - cw) + kCons * i;
        if (staged) {
          vreg[i] = rr < p.rank ? *reinterpret_cast<const uint4 *>(vs + rr * kSlab + 8 * lane)
                                : make_uint4(0u, 0u, 0u, 0u);
        } else {
          vreg[i] = make_uint4(0u, 0u, 0u, 0u);
          if (rr < p.rank && c0 < p.K)
            vreg[i] = *reinterpret_cast<const uint4 *>(p.V + (size_t)rr * p.K + c0);
        }
      }
#pragma unroll
      for (int tok = 0; tok < T; ++tok) {
        float xv[8];
        if (c0 < p.K) {
          const uint4 sg = *reinterpret_cast<const uint4 *>(xi + (size_t)tok * p.K + c0);
          const uint32_t sw[4] = {sg.x, sg.y, sg.z, sg.w};
          const float sc = xsc[tok * KG + c0 / 64];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int pp = seg_pos(j);
            const int16_t h = (int16_t)((sw[pp >> 1] >> (16 * (pp & 1))) & 0xFFFF);
            xv[j] = (float)h * sc;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) xv[j] = 0.0f;
        }
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int rr = (kCons - 1 - cw) + kCons * i;
          if (rr >= p.rank) break;
          const uint32_t w[4] = {vreg[i].x, vreg[i].y, vreg[i].z, vreg[i].w};
          float d = 0.0f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            d = fmaf(bf16_bits_to_f32(w[q] & 0xFFFFu), xv[2 * q], d);
            d = fmaf(bf16_bits_to_f32(w[q] >> 16), xv[2 * q + 1], d);
          }
#pragma unroll
          for (int o = 16; o; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
          if (lane == 0) p.tpart[((size_t)s * p.rank + rr) * p.T + tok] = d;
        }
      }
    }

  // ----------------------------------- units -----------------------------------
  // warp w takes a contiguous range; lane (r, h) = row r, half h of the unit.
  // Segments (a column group or salient chunk of one tile) are numbered by
  // key - key(u0); a warp flushes its partial at each segment change.
  const int r = lane & 15, h = lane >> 4;
  const int key0 = row_unit(u0, G).key;
  const int k0 = (cw * nu) / kCons, k1 = ((cw + 1) * nu) / kCons;
  float acc[T];
#pragma unroll
  for (int tok = 0; tok < T; ++tok) acc[tok] = 0.0f;
  int scur = k0 < k1 ? row_unit(u0 + k0, G).key - key0 : 0, slot_i = 0;
  if (lane == 0) {
    wt[2 * cw] = scur;
    wt[2 * cw + 1] = k0 < k1 ? row_unit(u0 + k1 - 1, G).key - key0 : scur - 1;
  }
  auto flush = [&]() {
#pragma unroll
    for (int tok = 0; tok < T; ++tok) {
      const float v = acc[tok] + __shfl_xor_sync(0xffffffffu, acc[tok], 16);
      if (h == 0) red[((cw * kRowSlots + slot_i) * T + tok) * 16 + r] = v;
      acc[tok] = 0.0f;
    }
  };
  bool ok = x_ok;
  RowUnit ru = row_unit(u0 + k0, G);
  for (int k = k0; k < k1 && ok; ++k, row_unit_next(ru, G)) {
    const int u = u0 + k;
    if (ru.key - key0 != scur) {
      flush();
      ++slot_i;
      scur = ru.key - key0;
    }
    if (!mbar_wait(&bars[k], 0)) { ok = false; break; }
    const uint8_t *row = us + k * kRowUnit + r * 128;
    if (!ru.q8) {
      const int j = ru.j;
      const uint16_t *sb = s4s + k * 128 + r * 8 + 4 * (j & 1) + 2 * h;
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const int gcol = 4 * j + 2 * h + gi;
        if (64 * gcol >= p.K) break;
        const int c0 = 4 * h + 2 * gi;
        const uint4 wa = *reinterpret_cast<const uint4 *>(row + ((c0 ^ (r & 7)) << 4));
        const uint4 wb = *reinterpret_cast<const uint4 *>(row + (((c0 + 1) ^ (r & 7)) << 4));
        const uint32_t wd[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
        // even columns (low nibbles) as bytes q + 8; odd columns (high
        // nibbles) masked in place, which as signed bytes are exactly 16 q
        uint32_t L[8], H[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          L[i] = lop3_splice(wd[i], 0x0F0F0F0Fu, 0x08080808u);
          H[i] = wd[i] & 0xF0F0F0F0u;
        }
        const float s4v = bf16_bits_to_f32(sb[gi]);
#pragma unroll
        for (int tok = 0; tok < T; ++tok) {
          const uint4 *xr = reinterpret_cast<const uint4 *>(xi + (size_t)tok * p.K + 64 * gcol);
          int d0 = 0, d1 = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint4 sg = xr[i];
            d0 = dp2a_lo(sg.x, L[i], d0);
            d0 = dp2a_hi(sg.y, L[i], d0);
            d1 = dp2a_lo(sg.z, H[i], d1);
            d1 = dp2a_hi(sg.w, H[i], d1);
          }
          const int dq = d0 - 8 * xsum[tok * KG + gcol] + (d1 >> 4);
          acc[tok] = fmaf(s4v * xsc[tok * KG + gcol], (float)dq, acc[tok]);
        }
      }
    } else {
      const int slot = u - q8first, cs = ru.j - jj0;
      // a full unit is 128 B per row in 128B-swizzled chunks; a narrower one
      // (QW = n_sal < 128) is QW bytes per row, unswizzled
      const uint8_t *qrow = us + k * kRowUnit + r * p.QW;
      uint32_t wd[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ch = 4 * h + i;
        uint4 w4 = make_uint4(0u, 0u, 0u, 0u);
        if (p.QW == 128)
          w4 = *reinterpret_cast<const uint4 *>(row + ((ch ^ (r & 7)) << 4));
        else if (16 * ch < p.QW)
          w4 = *reinterpret_cast<const uint4 *>(qrow + 16 * ch);
        wd[4 * i] = w4.x; wd[4 * i + 1] = w4.y; wd[4 * i + 2] = w4.z; wd[4 * i + 3] = w4.w;
      }
      const float s8v = bf16_bits_to_f32(s8s[slot * 64 + r]);
#pragma unroll
      for (int tok = 0; tok < T; ++tok) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(xs + ((size_t)cs * T + tok) * 128 + 64 * h);
        int d = 0, d1 = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 sg = xr[i];          // entries 8i .. 8i+7 of this half
          d = dp2a_lo(sg.x, wd[2 * i], d);
          d = dp2a_hi(sg.y, wd[2 * i], d);
          d1 = dp2a_lo(sg.z, wd[2 * i + 1], d1);
          d1 = dp2a_hi(sg.w, wd[2 * i + 1], d1);
        }
        acc[tok] = fmaf(s8v * xss[cs * T + tok], (float)(d + d1), acc[tok]);
      }
    }
  }
  if (k0 < k1) flush();
  consumer_sync();

  // one partial per segment: the warps' pieces summed in warp order, stored
  // in the segment's slot (2g or 2g + 1 for a column group, 2 ng + chunk for
  // a salient chunk)
  const int nseg = row_unit(u1 - 1, G).key - key0 + 1;
  const int nq4seg = G.ng * G.ntile;
  for (int i = ctid; i < nseg * T * 16; i += kConsThreads) {
    const int rr = i & 15, tok = (i >> 4) % T, sg = (i >> 4) / T;
    const int key = key0 + sg;
    int slot, t, zero_slot = -1;
    if (key < nq4seg) {
      const int g = key / G.ntile;
      t = key - g * G.ntile;
      int Sg;
      const int uf = seg_first(g, t, G, &Sg);
      const bool first = uf >= u0;
      slot = 2 * g + (first ? 0 : 1);
      if (first && uf + Sg <= u1) zero_slot = 2 * g + 1;      // whole segment here
    } else {
      const int v = key - nq4seg;
      t = v % G.ntile;
      slot = 2 * G.ng + v / G.ntile;
    }
    const int m = t * 16 + rr;
    if (m >= p.M) continue;
    float v = 0.0f;
    for (int w = 0; w < kCons; ++w) {
      const int sa = wt[2 * w], sb = wt[2 * w + 1];
      if (sg >= sa && sg <= sb) v += red[((w * kRowSlots + (sg - sa)) * T + tok) * 16 + rr];
    }
    p.part[((size_t)slot * p.T + tok) * p.M + m] = v;
    if (zero_slot >= 0) p.part[((size_t)zero_slot * p.T + tok) * p.M + m] = 0.0f;
  }
}

// ---------------------------------------------------------------- host ---
namespace {

struct RowPlan {
  RowGeom G;
  int units, grid, upc_max, maxq8, nscr, nslots;
  RowLayout L;
  bool ok;
};

int row_qw(int n_sal) { return n_sal >= 128 ? 128 : n_sal; }

// S slabs per column group; a segment of S units must not outgrow the
// smallest CTA share, so that at most two CTAs meet it.
RowGeom row_geom(int M, int K, int n_sal, int S) {
  RowGeom G;
  G.ntile = (M + 15) / 16;
  G.nslab = (K + kSlab - 1) / kSlab;
  G.S = std::max(1, std::min(S, G.nslab));
  G.ng = (G.nslab + G.S - 1) / G.S;
  G.Slast = G.nslab - (G.ng - 1) * G.S;
  G.nq4 = G.ntile * G.nslab;
  G.nq8u = n_sal > 0 ? (n_sal + row_qw(n_sal) - 1) / row_qw(n_sal) : 0;
  return G;
}

RowPlan row_plan(int M, int K, int block, int n_sal, int rank, int T, int nsm) {
  RowPlan d{};
  d.G = row_geom(M, K, n_sal, kRowGroupSlabs);
  d.units = d.G.nq4 + d.G.nq8u * d.G.ntile;      // does not depend on S
  int grid = std::min(d.units, nsm);
  while ((d.units + grid - 1) / grid > kRowMaxUnits) grid += std::max(1, grid / 4);
  d.grid = std::min(grid, d.units);
  d.upc_max = (d.units + d.grid - 1) / d.grid;
  d.G = row_geom(M, K, n_sal, std::min(kRowGroupSlabs, d.units / d.grid));
  const RowGeom &G = d.G;
  d.nslots = 2 * G.ng + G.nq8u;
  d.maxq8 = 0;
  for (int c = 0; c < d.grid; ++c) {
    const long long u0 = (long long)c * d.units / d.grid, u1 = (long long)(c + 1) * d.units / d.grid;
    d.maxq8 = std::max(d.maxq8, (int)std::max(0LL, u1 - std::max(u0, (long long)G.nq4)));
  }
  auto al = [](long long v) { return (int)((v + 127) / 128 * 128); };
  RowLayout &L = d.L;
  long long off = 0;
  auto put = [&](int &field, long long bytes) { field = (int)off; off += al(bytes); };
  put(L.units, (long long)d.upc_max * kRowUnit);
  put(L.s4, (long long)d.upc_max * 256);
  put(L.x, (long long)T * K * 2);
  put(L.xsc, (long long)T * (K / 64) * 4);
  put(L.xsum, (long long)T * (K / 64) * 4);
  put(L.xs, (long long)d.maxq8 * T * 256);
  put(L.xss, (long long)d.maxq8 * T * 4);
  put(L.sidx, (long long)d.maxq8 * 512);
  put(L.s8, (long long)d.maxq8 * 128);
  put(L.red, (long long)kRowWarps * kRowSlots * T * 16 * 4);
  put(L.wt, kRowWarps * 8);
  put(L.slist, (long long)(kRowMaxSlabMask + 1 + G.nslab) * 4);
  put(L.vs, (long long)rank * kSlab * 2 + 16);
  // FWHT scratch: as many 16-thread groups as fit (whole warps), at most one
  // per consumer thread group
  {
    const int P = block / 16, gpw = 32 / P, elems = 16 * (P + 1) + 1;
    const long long used = off + al((long long)(d.upc_max + 3) * 8) + 1024;
    int n = std::min({G.nslab * (kSlab / block) * T, kConsThreads / P,
                      (int)std::max(0LL, (kSmemLimit - used) / (elems * 4))});
    n = n / gpw * gpw;
    d.nscr = std::max(n, gpw);
    put(L.scr, (long long)d.nscr * elems * 4);
  }
  put(L.bars, (long long)(d.upc_max + 3) * 8);
  L.total = (int)std::min<long long>(off + 1024, 1LL << 30);
  // tensor-map boxes must not be wider than the rows they cut; the slab mask
  // covers K <= 65536
  d.ok = off + 1024 <= kSmemLimit && d.upc_max <= kRowMaxUnits && K >= 256 &&
         G.nslab <= 32 * kRowMaxSlabMask && (long long)d.units * 2 < (1LL << 31);
  return d;
}

}  // namespace

// Partial slots the column-group path writes per output, bounded for any
// group size (one slab per group at worst).
size_t decode_row_slices(int K, int n_sal) {
  const RowGeom G = row_geom(16, K, n_sal, 1);
  return (size_t)(2 * G.ng + G.nq8u);
}

// Returns cudaErrorNotSupported (with nothing launched) when the shape does
// not fit this path's shared-memory plan.
cudaError_t launch_decode_row(const ForwardArgs &a, cudaStream_t st, Launcher &Lc) {
  if (a.T < 1 || a.T > 2) return cudaErrorNotSupported;
  const RowPlan d = row_plan(a.M, a.K, a.block, a.n_sal, a.rank, a.T, sm_count());
  if (!d.ok) return cudaErrorNotSupported;
  RowParams p;
  p.M = a.M; p.K = a.K; p.T = a.T; p.n_sal = a.n_sal; p.rank = a.rank; p.block = a.block;
  p.G = d.G;
  p.units = d.units; p.grid = d.grid; p.upc_max = d.upc_max; p.maxq8 = d.maxq8; p.nscr = d.nscr;
  p.c = (float)sqrt(1.0 / (double)a.block);
  p.QW = row_qw(a.n_sal);
  p.s4 = a.s4; p.sal_idx = a.sal_idx; p.s8 = a.s8; p.V = a.V; p.x = a.x;
  p.L = d.L;
  char *ws = static_cast<char *>(a.workspace);
  size_t off = 0;
  auto take = [&](size_t b) { char *q = ws + off; off += (b + 255) & ~(size_t)255; return q; };
  p.part = reinterpret_cast<float *>(take(decode_row_slices(a.K, a.n_sal) * a.T * a.M * 4));
  p.tpart = reinterpret_cast<float *>(take((size_t)d.G.nslab * a.rank * a.T * 4 + 16));

  CUtensorMap mq4, ms4, mq8;
  if (encode_tmap_2d(&mq4, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q4, (uint64_t)a.K / 2, (uint64_t)a.M,
                     (uint64_t)a.K / 2, 128, 16, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  p.s4_tma = (a.K % 512 == 0) && ((uintptr_t)a.s4 % 16 == 0);
  ms4 = mq4;
  if (p.s4_tma && encode_tmap_2d(&ms4, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.s4, (uint64_t)a.K / 64,
                                 (uint64_t)a.M, (uint64_t)a.K / 32, 8, 16,
                                 CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
    p.s4_tma = 0;
  // s8 as one row of M BF16 values (the row stride is never stepped)
  CUtensorMap ms8 = mq4;
  if (a.n_sal > 0) {
    const CUresult r = encode_tmap_2d(&ms8, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.s8, (uint64_t)a.M, 1,
                                      ((uint64_t)a.M * 2 + 15) / 16 * 16, 16, 1,
                                      CU_TENSOR_MAP_SWIZZLE_NONE);
    if (r != CUDA_SUCCESS) {
      set_last_error("decode: s8 tensor map rejected (CUresult " + std::to_string((int)r) + ")");
      return cudaErrorInvalidValue;
    }
  }
  mq8 = mq4;
  if (a.n_sal > 0 &&
      encode_tmap_2d(&mq8, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q8, (uint64_t)a.n_sal, (uint64_t)a.M,
                     (uint64_t)a.n_sal, (uint32_t)p.QW, 16,
                     p.QW == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE) !=
          CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // V [rank][K] BF16, one slab (256 columns x rank rows) per box
  CUtensorMap mv = mq4;
  if (a.rank > 0 &&
      encode_tmap_2d(&mv, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.V, (uint64_t)a.K, (uint64_t)a.rank,
                     (uint64_t)a.K * 2, kSlab, (uint32_t)a.rank, CU_TENSOR_MAP_SWIZZLE_NONE) !=
          CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  const dim3 grid(d.grid), block(kRowThreads);
  const size_t smem = d.L.total;
  cudaError_t e;
  if (a.block == 256)
    e = a.T == 1 ? Lc.launch("dec_row", dec_row_kernel<256, 1>, grid, block, smem, st, true, mq4, ms4, mq8, ms8, mv, p)
                 : Lc.launch("dec_row", dec_row_kernel<256, 2>, grid, block, smem, st, true, mq4, ms4, mq8, ms8, mv, p);
  else
    e = a.T == 1 ? Lc.launch("dec_row", dec_row_kernel<128, 1>, grid, block, smem, st, true, mq4, ms4, mq8, ms8, mv, p)
                 : Lc.launch("dec_row", dec_row_kernel<128, 2>, grid, block, smem, st, true, mq4, ms4, mq8, ms8, mv, p);
  if (e != cudaSuccess) return e;

  DecodeParams tp{};
  tp.M = a.M; tp.K = a.K; tp.T = a.T; tp.n_sal = a.n_sal; tp.rank = a.rank; tp.block = a.block;
  tp.nslab = d.G.nslab;
  tp.U = a.U; tp.bias = a.bias; tp.y = a.y; tp.y_bf16 = a.y_bf16;
  tp.part = p.part; tp.tpart = p.tpart;
  tp.nslices = d.nslots;
  return Lc.launch("dec_tail", dec_tail_kernel, dim3((a.M + kTailThreads / 4 - 1) / (kTailThreads / 4), a.T),
                   dim3(kTailThreads), 0, st, true, tp);
}

cudaError_t prepare_decode_row_kernels() {
  cudaError_t e;
  for (const void *f : {(const void *)dec_row_kernel<256, 1>, (const void *)dec_row_kernel<256, 2>,
                        (const void *)dec_row_kernel<128, 1>, (const void *)dec_row_kernel<128, 2>}) {
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit)) !=
        cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

}  // namespace dvssq
