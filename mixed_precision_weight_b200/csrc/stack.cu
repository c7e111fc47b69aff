// One token through a stack of gated-GELU MLP blocks ("Myric/Spark-X2.5-4B-
// GGUF", "The model": GELU FFN; "Spark-X2.5-4B-ASHQ1-GGUF", "Architecture":
// ffn_gate / ffn_up / ffn_down), every projection a DV-SSQ layer (MiniCPM5-
// 2B-Hadamard-GSQ card, §2, with the Spark card's INT8 salient tier), in ONE
// persistent cooperative kernel:
//
//     g = RN_bf16(gate(x)),  u = RN_bf16(up(x)),  h = RN_bf16(gelu(g) u),
//     x <- RN_bf16(down(h)),   layer after layer.
//
// At one token every projection is a pure weight stream, and what a chain
// of separate launches loses is the per-launch latency: the dependency wait,
// the activation rotation and the partial-sum tail of every matrix.  Here the
// weights of the whole stack stream without a break:
//
//   * CTA c (one per SM) owns fixed row ranges: rows [c I/G, (c+1) I/G) of
//     every gate and up matrix and [c H/G, (c+1) H/G) of every down matrix.
//     A row's dot product then lives in one CTA, gelu(g) u needs no exchange
//     (gate and up rows coincide), and the CTA writes its slice of h or x.
//   * Warp 0 streams the CTA's rows of every matrix of the stack, in order,
//     through a ring of shared-memory slots (bulk copies of q4, s4, q8 and U
//     rows per row tile).  Nothing it reads depends on activations, so it
//     runs ahead across layer boundaries while the consumers wait.
//   * The other 15 (consumer) warps run two phases per block, each ending in
//     a grid barrier: gate+up (x -> h) and down (h -> x).  After a barrier every CTA
//     reads the whole input vector, rotates it (one warp per Hadamard block,
//     FP32 butterflies in registers and shuffles) into int16 with one scale
//     per 64 columns, requantises the salient entries per 32-entry chunk, and
//     runs its rows as exact int32 dot products by DP2A: even columns as
//     bytes q + 8 (minus 8 times the unit's even-column activation sum), odd
//     columns as the high nibble masked in place, a signed byte equal to
//     16 q (the sum divided by 16 exactly); scaled per group in FP32.  The
//     row work is cut into items (rows x rounds of 32-column lane tasks) that
//     the warps take from a shared counter; the warp that completes a tile's
//     last item frees its ring slot, and a warp ahead of the ring waits for
//     its tile by the slot's tag as well as the mbarrier's parity.
//   * The rank-r term needs t = V (H x) = (V H) x for all of x.  With
//     (V H) precomputed once in FP32, each CTA adds the share of the entries
//     it produced, t_c = (V H)[:, own] x[own], at the end of the producing
//     phase; after the barrier the consumers of t sum the G shares in a fixed
//     order.  No extra barrier is needed for it.
//
// Every wait is bounded (mbarriers and the grid barrier by the library's
// wait limit); a timeout sets the device error word and every warp leaves at
// its next wait.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>
#include <type_traits>

namespace dvssq {

constexpr int kStkWarps = 16;
constexpr int kStkThreads = 32 * kStkWarps;
constexpr int kStkCons = kStkWarps - 1;           // consumer warps (warp 0 streams weights)
constexpr int kStkConsThreads = 32 * kStkCons;
constexpr int kStkMaxRank = 32;                   // rank <= 32: one U t term per lane
constexpr int kStkMaxSlots = 24;
constexpr int kStkShareRegs = 5;                 // t shares per lane and pair: G <= 160

__device__ __forceinline__ void stk_consumer_sync() {
  asm volatile("bar.sync 2, %0;" ::"n"(kStkConsThreads) : "memory");
}
// Barrier among consumer warps 1.. only: they prepare the next phase while
// consumer warp 0 waits at the grid barrier.
constexpr int kStkPrepThreads = kStkConsThreads - 32;
__device__ __forceinline__ void stk_prep_sync() {
  asm volatile("bar.sync 3, %0;" ::"n"(kStkPrepThreads) : "memory");
}

struct StackParams {
  const StackLayerDesc *layers;   // [L] in device memory
  int L, H, I, G;
  int tr_gu, tr_d;                // rows per tile of gate/up and of down
  int slot_bytes, nslots;
  int max_rank, max_nsal, rows_max, rounds_max;
  const uint16_t *x;              // BF16 [H]
  uint16_t *y;                    // BF16 [H]: the running hidden state, then the output
  uint16_t *h;                    // BF16 [I]
  float *tp;                      // t shares [3][kStkMaxRank][Gp]: gate, up, down
  unsigned int *gbar;             // grid barrier counter, zero at launch
  // shared-memory offsets from the 1024-aligned base
  int o_ring, o_full, o_empty, o_xi, o_xsc, o_xs8, o_xs, o_xss, o_sidx, o_t, o_s8, o_yv, o_vh,
      o_flag, o_grab, o_ph, o_ld, o_vhs, smem_total;
};

// Stride of the t shares of one (matrix, rank index) pair: G rounded up to
// whole 16-byte words, so that each pair's shares copy as 16-byte chunks.
__host__ __device__ constexpr int stk_gp(int G) { return (G + 3) & ~3; }

// Entries per matrix of the BF16 s8 staging: the own rows plus the partial
// 16-byte words at both ends, rounded up to whole words.
__host__ __device__ constexpr int stk_s8_stride(int rows_max) { return (rows_max + 16 + 7) & ~7; }

// Row range of CTA c among G for M rows.
__device__ __forceinline__ int stk_row(int c, int M, int G) {
  return (int)(((long long)c * M) / G);
}

// Position of column j (0..7) of an 8-column segment in the DP2A order
// {0, 2, 4, 6, 1, 3, 5, 7} of the stored int16 activations.
__device__ __forceinline__ int stk_seg_pos(int j) { return (j & 1) ? 4 + (j >> 1) : (j >> 1); }

__device__ __forceinline__ uint32_t stk_splice(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Bounded mbarrier wait that also gives up as soon as another warp of the CTA
// has flagged an abort.  Between polls the warp sleeps briefly, so that a
// waiting warp does not take issue slots from the warps that compute.
__device__ __forceinline__ bool stk_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64(), lim = wait_limit();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (clock64() - t0 > lim) {
      set_error(kErrWaitMbarrier);
      *abort = 1;
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// The same wait for a ring slot that also requires the slot's tile tag: the
// parity of an mbarrier cannot tell tile T from tile T - 2 NS, the tag can,
// so consumer warps may run ahead of the ring by more than a turn.  The
// producer writes a slot's tag only after the slot's previous tile was freed,
// and the tag is read (acquire) before the parity is tested: a tag equal to
// the wanted tile means the phases before it have completed, so the parity
// then names this tile's phase alone.
__device__ __forceinline__ int stk_tag_acquire(const int *tag) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];"
               : "=r"(v)
               : "r"(smem_u32(tag))
               : "memory");
  return v;
}

__device__ __forceinline__ bool stk_wait_tile(uint64_t *bar, uint32_t parity, const int *tag,
                                              int want, volatile int *abort) {
  auto ready = [&]() { return stk_tag_acquire(tag) == want && mbar_try_wait(bar, parity); };
  if (ready()) return true;
  const long long t0 = clock64(), lim = wait_limit();
  while (!ready()) {
    if (*abort) return false;
    if (clock64() - t0 > lim) {
      set_error(kErrWaitMbarrier);
      *abort = 1;
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// Activations in shared memory: 32-column units of int16 in four 16-byte
// chunks (8 columns each, DP2A order inside), chunk i of unit v stored at
// position i ^ ((v >> 1) & 3) so that lanes reading consecutive units hit
// distinct banks.
__device__ __forceinline__ int stk_chunk(int v, int i) { return i ^ ((v >> 1) & 3); }
__device__ __forceinline__ int stk_xpos(int col) {
  const int v = col >> 5;
  return 32 * v + 8 * stk_chunk(v, (col >> 3) & 3) + stk_seg_pos(col & 7);
}

struct StkPhase {
  int nm;                   // matrices of the phase (2: gate and up; 1: down)
  StackMatDesc m[2];
  int K, a, b, tr;          // input length, own rows [a, b), rows per tile (even)
  const uint16_t *src;      // input vector (BF16 [K])
  int tslot[2];             // t-share slot of each matrix
  // the matrices that consume this phase's output: their (V H) columns [a, b)
  // give this CTA's t shares
  int nout;
  const float *ovh[2];
  int oK[2], orank[2], oslot[2];
  // the rows' item plan (stk_plan_items): rows per item, items in all, and
  // per matrix its items, items per tile, tiles, round groups and rounds
  // per item
  int rg, total, tot[2], ipt[2], ntl[2], nrg[2], rr[2];
};

__device__ __forceinline__ void stk_cp_async4(void *smem, const void *gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void stk_cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void stk_cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void stk_cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// One item of a tile for one consumer warp: rows [RG gi, RG gi + RG) of the
// tile x rounds [RR rq, RR rq + RR), straight-line; a row past the tile
// repeats its last row and is masked when written.  Every operand comes in by
// value (no closure): the hot code keeps them in registers.
struct StkTileArgs {
  const uint8_t *q4s, *s4s, *q8s;
  const uint16_t *us, *xi, *xsm, *s8m;
  const int *xsu;
  const float *xsc, *xssm, *tvm;
  float *red;
  int kq, ks, nsal, nu4, nu8, rk, nr, nrg, ra, mi, rows_max, rounds_max;
};

template <int RGc, int RRc>
__device__ __forceinline__ void stk_item(const StkTileArgs a, int it, int lane) {
  const uint8_t *__restrict__ q4s = a.q4s;
  const uint8_t *__restrict__ s4s = a.s4s;
  const uint8_t *__restrict__ q8s = a.q8s;
  const uint16_t *__restrict__ us = a.us;
  const uint16_t *__restrict__ xi = a.xi;
  const uint16_t *__restrict__ xsm = a.xsm;
  const uint16_t *__restrict__ s8m = a.s8m;
  const int *__restrict__ xsu = a.xsu;
  const float *__restrict__ xsc = a.xsc;
  const float *__restrict__ xssm = a.xssm;
  const float *__restrict__ tvm = a.tvm;
  const int kq = a.kq, ks = a.ks, nsal = a.nsal, nu4 = a.nu4, nu8 = a.nu8, rk = a.rk;
  const int nr = a.nr, nrg = a.nrg;
  const int gi = it / nrg, rq = it - gi * nrg;
  const int r0 = gi * RGc;
  int rl[RGc];
  float acc[RGc];
#pragma unroll
  for (int ri = 0; ri < RGc; ++ri) {
    rl[ri] = min(r0 + ri, nr - 1);
    acc[ri] = 0.0f;
  }
#pragma unroll
  for (int u = 0; u < RRc; ++u) {
    const int task = 32 * (rq * RRc + u) + lane;
    float f[RGc];
    if (task < nu4) {
      const int v = task, g = v >> 1;
      uint4 xa[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        xa[i] = *reinterpret_cast<const uint4 *>(xi + 32 * v + 8 * stk_chunk(v, i));
      const int bias = 8 * xsu[v];
      const float sc = xsc[g];
#pragma unroll
      for (int ri = 0; ri < RGc; ++ri) {
        const uint4 w4 = *reinterpret_cast<const uint4 *>(q4s + (size_t)rl[ri] * kq + 16 * v);
        const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
        // even columns (low nibbles) as bytes q + 8; odd columns (high
        // nibbles) masked in place, which as signed bytes are exactly 16 q
        int de[2] = {0, 0}, dd[2] = {0, 0};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t L = stk_splice(wd[i], 0x0F0F0F0Fu, 0x08080808u);
          const uint32_t Hs = wd[i] & 0xF0F0F0F0u;
          de[i & 1] = __dp2a_lo((int)xa[i].x, (int)L, de[i & 1]);
          de[i & 1] = __dp2a_hi((int)xa[i].y, (int)L, de[i & 1]);
          dd[i & 1] = __dp2a_lo((int)xa[i].z, (int)Hs, dd[i & 1]);
          dd[i & 1] = __dp2a_hi((int)xa[i].w, (int)Hs, dd[i & 1]);
        }
        const float s4v =
            bf16_bits_to_f32(reinterpret_cast<const uint16_t *>(s4s + (size_t)rl[ri] * ks)[g]);
        f[ri] = s4v * sc * (float)((de[0] + de[1] - bias) + ((dd[0] + dd[1]) >> 4));
      }
    } else if (task < nu4 + nu8) {
      const int j = task - nu4;
      uint4 xa[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        xa[i] = *reinterpret_cast<const uint4 *>(xsm + 32 * j + 8 * stk_chunk(j, i));
      const float sc = xssm[j];
#pragma unroll
      for (int ri = 0; ri < RGc; ++ri) {
        const uint8_t *qr = q8s + (size_t)rl[ri] * nsal + 32 * j;
        const uint4 qa = *reinterpret_cast<const uint4 *>(qr);
        const uint4 qb = *reinterpret_cast<const uint4 *>(qr + 16);
        const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        int d[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          d[i] = __dp2a_lo((int)xa[i].x, (int)qw[2 * i], d[i]);
          d[i] = __dp2a_hi((int)xa[i].y, (int)qw[2 * i], d[i]);
          d[i] = __dp2a_lo((int)xa[i].z, (int)qw[2 * i + 1], d[i]);
          d[i] = __dp2a_hi((int)xa[i].w, (int)qw[2 * i + 1], d[i]);
        }
        f[ri] = bf16_bits_to_f32(s8m[a.ra + rl[ri]]) * sc * (float)((d[0] + d[1]) + (d[2] + d[3]));
      }
    } else {
#pragma unroll
      for (int ri = 0; ri < RGc; ++ri) f[ri] = 0.0f;
    }
#pragma unroll
    for (int ri = 0; ri < RGc; ++ri) acc[ri] += f[ri];
  }
  if (rq == 0 && lane < rk) {
#pragma unroll
    for (int ri = 0; ri < RGc; ++ri)
      acc[ri] = fmaf(bf16_bits_to_f32(us[rl[ri] * rk + lane]), tvm[lane], acc[ri]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
#pragma unroll
    for (int ri = 0; ri < RGc; ++ri) acc[ri] += __shfl_xor_sync(0xffffffffu, acc[ri], o);
  }
  if (lane == 0) {
#pragma unroll
    for (int ri = 0; ri < RGc; ++ri)
      if (r0 + ri < nr)
        a.red[((size_t)a.mi * a.rows_max + a.ra + r0 + ri) * a.rounds_max + rq] = acc[ri];
  }
}

// Rounds per item for a matrix of `rounds` 32-task rounds: three or four,
// as even as possible (3 for 3 rounds, 4 for 12, 3 for 9; 3 for one or two
// rounds, whose missing rounds are idle).  Two item shapes per row count
// keep the kernel's code small.
__host__ __device__ __forceinline__ int stk_rr(int rounds) {
  const int n = (rounds + 3) / 4;
  return max(3, (rounds + n - 1) / n);
}

// The item plan of a phase, computed once by the thread that writes its
// descriptor.  RG = 5 (or 4) rows per item where the tile's rows allow it
// and every matrix of the phase takes three-round items, else 2 (four item
// shapes in all).  Five-row items cut a gate+up phase of the Spark shapes
// (70 rows of each matrix per CTA) into 28 items, two even waves over the
// 15 consumer warps, where four-row items made 36 (a third wave for 6).
__device__ __forceinline__ void stk_plan_items(StkPhase &ph) {
  const int nrows = ph.b - ph.a;
  int RG = ph.tr % 5 == 0 ? 5 : ph.tr % 4 == 0 ? 4 : 2;
  for (int mi = 0; mi < ph.nm; ++mi)
    if (stk_rr((ph.m[mi].K / 32 + ph.m[mi].n_sal / 32 + 31) / 32) != 3) RG = 2;
  ph.rg = RG;
  ph.total = 0;
  for (int mi = 0; mi < 2; ++mi) {
    const bool on = mi < ph.nm;
    const int K = on ? ph.m[mi].K : 32, nsal = on ? ph.m[mi].n_sal : 0;
    const int rounds = (K / 32 + nsal / 32 + 31) / 32;
    ph.rr[mi] = stk_rr(rounds);
    ph.nrg[mi] = (rounds + ph.rr[mi] - 1) / ph.rr[mi];
    ph.ntl[mi] = on ? (nrows + ph.tr - 1) / ph.tr : 0;
    ph.ipt[mi] = (ph.tr / RG) * ph.nrg[mi];
    const int nl = nrows - (ph.ntl[mi] - 1) * ph.tr;
    ph.tot[mi] = on ? (ph.ntl[mi] - 1) * ph.ipt[mi] + ((nl + RG - 1) / RG) * ph.nrg[mi] : 0;
    ph.total += ph.tot[mi];
  }
}

template <int B>
__global__ void __launch_bounds__(kStkThreads, 1) mlp_stack_kernel(const StackParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *ring = base + p.o_ring;
  uint64_t *full = reinterpret_cast<uint64_t *>(base + p.o_full);
  uint64_t *empty = reinterpret_cast<uint64_t *>(base + p.o_empty);
  uint16_t *xi = reinterpret_cast<uint16_t *>(base + p.o_xi);   // [Kmax]: BF16 in, int16 out
  float *xsc = reinterpret_cast<float *>(base + p.o_xsc);       // [Kmax / 64]
  int *xsu = reinterpret_cast<int *>(base + p.o_xs8);           // [Kmax / 32] unit sums
  uint16_t *xsal = reinterpret_cast<uint16_t *>(base + p.o_xs); // [2][max_nsal] int16
  float *xss = reinterpret_cast<float *>(base + p.o_xss);       // [2][max_nsal / 32]
  int *sidx = reinterpret_cast<int *>(base + p.o_sidx);         // [2][max_nsal]
  float *tv = reinterpret_cast<float *>(base + p.o_t);          // [2][kStkMaxRank]
  uint16_t *s8c = reinterpret_cast<uint16_t *>(base + p.o_s8);  // [2][s8_stride] BF16
  float *red = reinterpret_cast<float *>(base + p.o_yv);        // [2][rows_max][rounds_max]
  float *vals = reinterpret_cast<float *>(base + p.o_vh);       // [rows_max] produced values
  volatile int *abort = reinterpret_cast<volatile int *>(base + p.o_flag);
  int *s_grab = reinterpret_cast<int *>(base + p.o_grab);        // next item of the phase
  StkPhase *sph = reinterpret_cast<StkPhase *>(base + p.o_ph);  // the current phase
  StackLayerDesc *sld = reinterpret_cast<StackLayerDesc *>(base + p.o_ld);  // layers l, l + 1 at [l & 1]
  int *s_done = s_grab + 1;                                       // [nslots] items done per slot
  int *s_tag = s_done + kStkMaxSlots;                             // [nslots] tile held per slot

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = p.G;
  const int gu_a = stk_row(c, p.I, G), gu_b = stk_row(c + 1, p.I, G);
  const int d_a = stk_row(c, p.H, G), d_b = stk_row(c + 1, p.H, G);
  const int NS = p.nslots;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      s_done[s] = 0;
      s_tag[s] = -1;
    }
    fence_mbarrier_init();
    *abort = 0;
    *s_grab = 0;
  }
  __syncthreads();

  // ------------------------------- weight stream -------------------------------
  if (warp == 0) {
    if (lane == 0) {
      uint32_t seq = 0;
      bool ok = true;
      for (int l = 0; l < p.L && ok; ++l)
        for (int mi = 0; mi < 3 && ok; ++mi) {
          const StackMatDesc m = p.layers[l].m[mi];
          const int a = mi < 2 ? gu_a : d_a, b = mi < 2 ? gu_b : d_b;
          const int tr = mi < 2 ? p.tr_gu : p.tr_d;
          const uint32_t kq = (uint32_t)m.K / 2, ks = (uint32_t)m.K / 32;
          for (int i0 = a; i0 < b; i0 += tr, ++seq) {
            const uint32_t nr = (uint32_t)min(tr, b - i0);
            const int s = (int)(seq % (uint32_t)NS);
            const uint32_t n = seq / (uint32_t)NS;
            if (n > 0 && !stk_wait(&empty[s], (n - 1) & 1u, abort)) {
              ok = false;
              break;
            }
            uint8_t *dst = ring + (size_t)s * p.slot_bytes;
            const uint32_t bq = nr * kq, bs = nr * ks, b8 = nr * (uint32_t)m.n_sal;
            const uint32_t bu = nr * (uint32_t)m.r * 2u;
            *(volatile int *)&s_tag[s] = (int)seq;
            mbar_arrive_expect_tx(&full[s], bq + bs + b8 + bu);
            bulk_g2s(dst, m.q4 + (size_t)i0 * kq, bq, &full[s]);
            bulk_g2s(dst + bq, reinterpret_cast<const uint8_t *>(m.s4) + (size_t)i0 * ks, bs,
                     &full[s]);
            if (b8) bulk_g2s(dst + bq + bs, m.q8 + (size_t)i0 * m.n_sal, b8, &full[s]);
            if (bu) bulk_g2s(dst + bq + bs + b8, m.U + (size_t)i0 * m.r, bu, &full[s]);
          }
        }
      // copies still in flight land before the CTA may exit
      const uint32_t issued = seq;
      for (uint32_t q = issued > (uint32_t)NS ? issued - (uint32_t)NS : 0u; q < issued; ++q)
        mbar_wait(&full[q % (uint32_t)NS], (q / (uint32_t)NS) & 1u);
    }
    return;
  }

  // --------------------------------- consumers ---------------------------------
  const int ctid = tid - 32, cw = warp - 1;
  const unsigned int err0 = *(volatile uint32_t *)&g_dvssq_error;
  uint32_t seq = 0;            // ring position, in step with the producer
  unsigned int nbar = 0;       // grid barriers passed
  const int rows_max = p.rows_max, rounds_max = p.rounds_max;
  // per-matrix BF16 staging of s8: 16-byte words covering the own rows, so a
  // multiple of 8 entries (each slice starts 16-byte aligned)
  const int s8_stride = stk_s8_stride(rows_max);
  volatile int *s_live = abort + 1;
  float *vhs = reinterpret_cast<float *>(base + p.o_vhs);       // (V H) columns of own outputs

  // Split grid barrier: a CTA arrives as soon as its outputs are written,
  // prefetches what the next phase needs from the weights, then waits.
  auto grid_arrive = [&]() {
    ++nbar;
    stk_consumer_sync();
    if (ctid == 0 && *abort == 0) {
      __threadfence();
      atomicAdd(p.gbar, 1u);
    }
  };
  auto grid_wait = [&]() -> bool {
    if (ctid == 0 && *abort == 0 && !counter_wait(p.gbar, nbar * (unsigned int)G, err0))
      *abort = 1;
    // one thread decides, so that every consumer warp takes the same branches
    if (ctid == 0) *s_live = *abort == 0;
    stk_consumer_sync();
    return *s_live != 0;
  };

  // Layer descriptors of layers l and l + 1 sit in shared memory (slot l & 1),
  // copied by cp.async a phase ahead, so that building a phase descriptor at
  // a grid barrier reads no global memory.
  static_assert(sizeof(StackLayerDesc) % 16 == 0, "layer descriptors copy as 16-byte chunks");
  auto fetch_layer = [&](int l) {
    constexpr int n16 = (int)(sizeof(StackLayerDesc) / 16);
    if (ctid < n16)
      stk_cp_async16(reinterpret_cast<uint4 *>(sld + (l & 1)) + ctid,
                     reinterpret_cast<const uint4 *>(p.layers + l) + ctid);
    stk_cp_async_commit();
  };

  // phase descriptors: layer l, kind 0 = gate and up (x -> h), 1 = down (h -> x).
  // One thread writes the descriptor to shared memory and the consumers read
  // it there: a per-thread copy would live in local memory, whose lines the
  // small L1 (shared memory takes the rest) loses to L2 between uses.
  // `prep`: written by the first thread of consumer warp 1 and published to
  // warps 1.. only (the grid-barrier path); else by consumer thread 0 to all.
  auto set_phase = [&](int l, int kind, bool prep) {
    if (ctid == (prep ? 32 : 0)) {
      StkPhase &ph = *sph;
      const StackLayerDesc *Ld = sld + (l & 1);
      const StackLayerDesc *Ln = sld + ((l + 1) & 1);
      if (kind == 0) {
        ph.nm = 2;
        ph.m[0] = Ld->m[0];
        ph.m[1] = Ld->m[1];
        ph.K = p.H;
        ph.a = gu_a;
        ph.b = gu_b;
        ph.tr = p.tr_gu;
        ph.src = l == 0 ? p.x : p.y;
        ph.tslot[0] = 0;
        ph.tslot[1] = 1;
        ph.nout = 1;
        ph.ovh[0] = Ld->m[2].vh;
        ph.oK[0] = Ld->m[2].K;
        ph.orank[0] = Ld->m[2].r;
        ph.oslot[0] = 2;
      } else {
        ph.nm = 1;
        ph.m[0] = Ld->m[2];
        ph.K = p.I;
        ph.a = d_a;
        ph.b = d_b;
        ph.tr = p.tr_d;
        ph.src = p.h;
        ph.tslot[0] = 2;
        ph.nout = l + 1 < p.L ? 2 : 0;
        for (int j = 0; j < ph.nout; ++j) {
          ph.ovh[j] = Ln->m[j].vh;
          ph.oK[j] = Ln->m[j].K;
          ph.orank[j] = Ln->m[j].r;
          ph.oslot[j] = j;
        }
      }
      stk_plan_items(ph);
    }
    if (prep) stk_prep_sync();
    else stk_consumer_sync();
  };

  // weight-side data of a phase, loaded while the grid barrier is pending:
  // INT8 scales of the own rows, salient indices, (V H) columns for the t shares
  // issued by threads t0.. of the consumers, nth of them
  auto prefetch = [&](const StkPhase &ph, int t0, int nth) {
    const int n = ph.b - ph.a, tt = ctid - t0;
    for (int mi = 0; mi < ph.nm; ++mi) {
      const StackMatDesc &m = ph.m[mi];
      if (m.n_sal == 0) continue;
      // the 16-byte words of s8 that hold rows [a, b) (M is a multiple of 8)
      const int w0 = ph.a >> 3, w1 = (ph.b + 7) >> 3;
      for (int w = w0 + tt; w < w1; w += nth)
        stk_cp_async16(s8c + mi * s8_stride + 8 * (w - w0), m.s8 + 8 * w);
      for (int e = 4 * tt; e < m.n_sal; e += 4 * nth)
        stk_cp_async16(sidx + mi * p.max_nsal + e, m.sal_idx + e);
    }
    int off = 0;
    for (int j = 0; j < ph.nout; ++j) {
      for (int q = tt; q < ph.orank[j] * n; q += nth) {
        const int k = q / n, i = q - k * n;
        stk_cp_async4(vhs + off + q, ph.ovh[j] + (size_t)k * ph.oK[j] + ph.a + i);
      }
      off += ph.orank[j] * n;
    }
    stk_cp_async_commit();
  };

  // this CTA's t shares for the consumers of its outputs vals[0..n)
  auto t_share_out = [&](const StkPhase &ph) {
    const int n = ph.b - ph.a;
    int off = 0;
    for (int j = 0; j < ph.nout; ++j) {
      for (int k = cw; k < ph.orank[j]; k += kStkCons) {
        const float *row = vhs + off + k * n;
        float s = 0.0f;
        for (int i = lane; i < n; i += 32) s = fmaf(row[i], vals[i], s);
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) p.tp[((size_t)ph.oslot[j] * kStkMaxRank + k) * stk_gp(G) + c] = s;
      }
      off += ph.orank[j] * n;
    }
  };

  // ---- one phase: activations in, the CTA's rows of one or two matrices out
  auto run_phase = [&](const StkPhase &ph) {
    const int K = ph.K, nrows = ph.b - ph.a;
    if (ctid == 0) *s_grab = 0;    // the previous phase's rows ended before its last barrier
    // The input vector comes in by cp.async (the rotation waits for it); the
    // G shares of each (matrix, rank index) pair are loaded into registers
    // now and summed after the rotation and the salient step, so that their
    // latency hides behind both.  Both were written by other CTAs before the
    // grid barrier: the loads read L2 (.cg).  Warp cw takes the pairs
    // q = cw + kStkCons i; its lanes hold the shares at lane + 32 u.
    const int r0m = ph.m[0].r, npair = r0m + (ph.nm > 1 ? ph.m[1].r : 0);
    const int Gp = stk_gp(G);
    for (int i = ctid; i < K / 8; i += kStkConsThreads) stk_cp_async16(xi + 8 * i, ph.src + 8 * i);
    stk_cp_async_commit();
    constexpr int QW = (2 * kStkMaxRank + kStkCons - 1) / kStkCons;   // pairs per warp
    float tsv[QW][kStkShareRegs];
#pragma unroll
    for (int i = 0; i < QW; ++i) {
      const int q = cw + kStkCons * i;
      const int mi = q < r0m ? 0 : 1, k = q - (mi ? r0m : 0);
      const float *src = p.tp + ((size_t)ph.tslot[mi] * kStkMaxRank + k) * Gp;
#pragma unroll
      for (int u = 0; u < kStkShareRegs; ++u) {
        const int j = lane + 32 * u;
        tsv[i][u] = (q < npair && j < G) ? __ldcg(src + j) : 0.0f;
      }
    }
    stk_cp_async_wait_all();             // the prefetched s8 and salient indices, and x
    stk_consumer_sync();

    // rotate x: BF16 in, int16 (unit/chunk layout) with one scale per 64
    // columns.  One warp per Hadamard block: lane l holds the E = B/32
    // consecutive columns [E l, E l + E); the butterflies inside a lane run
    // in registers, the ones across lanes (index bits log2 E and up) by
    // shuffles.  The block is read whole before its int16 form is written
    // back in place (both stay inside the block).
    {
      constexpr int E = B / 32;                // columns per lane: 8 or 4
      constexpr int LPG = 64 / E;              // lanes per 64-column group: 8 or 16
      constexpr int LPU = 32 / E;              // lanes per 32-column unit: 4 or 8
      const int nblk = K / B;
      const float cb = B == 256 ? 0.0625f : 0.08838834764831845f;
      for (int kb = cw; kb < nblk; kb += kStkCons) {
        const uint16_t *blk = xi + (size_t)kb * B + E * lane;
        float v[E];
        if constexpr (E == 8) {
          const uint4 w = *reinterpret_cast<const uint4 *>(blk);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16_bits_to_f32(ww[i] & 0xFFFFu);
            v[2 * i + 1] = bf16_bits_to_f32(ww[i] >> 16);
          }
        } else {
          const uint2 w = *reinterpret_cast<const uint2 *>(blk);
          v[0] = bf16_bits_to_f32(w.x & 0xFFFFu);
          v[1] = bf16_bits_to_f32(w.x >> 16);
          v[2] = bf16_bits_to_f32(w.y & 0xFFFFu);
          v[3] = bf16_bits_to_f32(w.y >> 16);
        }
        __syncwarp();
#pragma unroll
        for (int h = 1; h < E; h <<= 1)
#pragma unroll
          for (int i = 0; i < E; ++i)
            if (!(i & h)) {
              const float a = v[i], b2 = v[i + h];
              v[i] = a + b2;
              v[i + h] = a - b2;
            }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const bool upper = (lane & o) != 0;
#pragma unroll
          for (int i = 0; i < E; ++i) {
            const float other = __shfl_xor_sync(0xffffffffu, v[i], o);
            v[i] = upper ? other - v[i] : v[i] + other;
          }
        }
        float mx = 0.0f;
#pragma unroll
        for (int j = 0; j < E; ++j) {
          v[j] *= cb;
          mx = fmaxf(mx, fabsf(v[j]));
        }
#pragma unroll
        for (int o = 1; o < LPG; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float inv = mx > 0.0f ? 32767.0f / mx : 0.0f;
        int q[E], sum = 0;      // sum over the even columns (their codes carry the +8)
#pragma unroll
        for (int j = 0; j < E; ++j) {
          q[j] = max(-32767, min(32767, __float2int_rn(v[j] * inv)));
          if (!(j & 1)) sum += q[j];
        }
#pragma unroll
        for (int o = 1; o < LPU; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const int col0 = kb * B + E * lane, vu = col0 >> 5, ci = (col0 >> 3) & 3;
        uint16_t *chunk = xi + 32 * vu + 8 * stk_chunk(vu, ci);
        // DP2A order inside the 8-column chunk: {0, 2, 4, 6, 1, 3, 5, 7}
        if constexpr (E == 8) {
          uint4 w;
          w.x = (uint32_t)(q[0] & 0xFFFF) | ((uint32_t)q[2] << 16);
          w.y = (uint32_t)(q[4] & 0xFFFF) | ((uint32_t)q[6] << 16);
          w.z = (uint32_t)(q[1] & 0xFFFF) | ((uint32_t)q[3] << 16);
          w.w = (uint32_t)(q[5] & 0xFFFF) | ((uint32_t)q[7] << 16);
          *reinterpret_cast<uint4 *>(chunk) = w;
        } else {
          // this lane holds columns 0..3 (lane even) or 4..7 (lane odd) of
          // the chunk: words x, z or y, w of it
          uint32_t *cw32 = reinterpret_cast<uint32_t *>(chunk) + (lane & 1);
          cw32[0] = (uint32_t)(q[0] & 0xFFFF) | ((uint32_t)q[2] << 16);
          cw32[2] = (uint32_t)(q[1] & 0xFFFF) | ((uint32_t)q[3] << 16);
        }
        if (lane % LPG == 0) xsc[col0 >> 6] = mx * (1.0f / 32767.0f);
        if (lane % LPU == 0) xsu[vu] = sum;
      }
    }
    stk_consumer_sync();

    // salient activations of each matrix, requantised per 32-entry chunk
    for (int mi = 0; mi < ph.nm; ++mi) {
      const int ns = ph.m[mi].n_sal;
      for (int j = cw; j < ns / 32; j += kStkCons) {
        const int col = sidx[mi * p.max_nsal + 32 * j + lane];
        float val = 0.0f;
        if (col >= 0 && col < K) val = (float)(int16_t)xi[stk_xpos(col)] * xsc[col >> 6];
        float mx = fabsf(val);
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float inv = mx > 0.0f ? 32767.0f / mx : 0.0f;
        const int qv = max(-32767, min(32767, __float2int_rn(val * inv)));
        xsal[mi * p.max_nsal + 32 * j + 8 * stk_chunk(j, lane >> 3) + (lane & 7)] =
            (uint16_t)(qv & 0xFFFF);
        if (lane == 0) xss[mi * (p.max_nsal / 32) + j] = mx * (1.0f / 32767.0f);
      }
    }
    // t = the sum of the G shares of each pair, in u order and then by a
    // fixed shuffle tree (deterministic)
#pragma unroll
    for (int i = 0; i < QW; ++i) {
      const int q = cw + kStkCons * i;
      float sum = 0.0f;
#pragma unroll
      for (int u = 0; u < kStkShareRegs; ++u) sum += tsv[i][u];
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0 && q < npair) {
        const int mi = q < r0m ? 0 : 1, k = q - (mi ? r0m : 0);
        tv[mi * kStkMaxRank + k] = sum;
      }
    }
    stk_consumer_sync();

    // The rows.  A lane task is 32 columns of q4 (or 32 salient entries of
    // q8) of one row; a round is 32 consecutive tasks.  An item is RG rows x
    // RR rounds of one tile (RG = 5 or 4 for three-round items when the
    // tile's rows allow it, else 2: stk_plan_items).  The consumer warps take
    // items from a shared counter in (matrix, tile, item) order, which is the
    // ring's order; the warp that completes a tile's last item frees its ring
    // slot.  A warp that takes an item of a tile whose slot still holds an
    // earlier tile waits for the slot's tag (stk_wait_tile).
    {
      const int RG = ph.rg, total = ph.total;
      const int tot0 = ph.tot[0], ntl0 = ph.ntl[0];
      for (;;) {
        int gx = 0;
        if (lane == 0) gx = atomicAdd(s_grab, 1);
        gx = __shfl_sync(0xffffffffu, gx, 0);
        if (gx >= total) break;
        const int mi = gx < tot0 ? 0 : 1;
        const int g = gx - (mi ? tot0 : 0);
        const int ipt = ph.ipt[mi];
        const int tile = g / ipt, it = g - tile * ipt;
        const uint32_t tseq = seq + (uint32_t)((mi ? ntl0 : 0) + tile);
        const int s = (int)(tseq % (uint32_t)NS);
        const bool got = __all_sync(
            0xffffffffu, stk_wait_tile(&full[s], (tseq / (uint32_t)NS) & 1u, s_tag + s, (int)tseq, abort));
        const int i0 = ph.a + tile * ph.tr;
        const int nr = min(ph.tr, ph.b - i0);
        const int nsal = ph.m[mi].n_sal, Km = ph.m[mi].K;
        const int nrg = ph.nrg[mi], rr = ph.rr[mi];
        const int kq = Km / 2, ks = Km / 32;
        const uint8_t *q4s = ring + (size_t)s * p.slot_bytes;
        const uint8_t *s4s = q4s + nr * kq, *q8s = s4s + nr * ks;
        StkTileArgs ta;
        ta.q4s = q4s; ta.s4s = s4s; ta.q8s = q8s;
        ta.us = reinterpret_cast<const uint16_t *>(q8s + nr * nsal);
        ta.xi = xi; ta.xsm = xsal + mi * p.max_nsal;
        ta.s8m = s8c + mi * s8_stride + (ph.a & 7);
        ta.xsu = xsu; ta.xsc = xsc; ta.xssm = xss + mi * (p.max_nsal / 32);
        ta.tvm = tv + mi * kStkMaxRank; ta.red = red;
        ta.kq = kq; ta.ks = ks; ta.nsal = nsal; ta.nu4 = Km / 32; ta.nu8 = nsal / 32;
        ta.rk = ph.m[mi].r;
        ta.nr = nr; ta.nrg = nrg; ta.ra = i0 - ph.a; ta.mi = mi;
        ta.rows_max = rows_max; ta.rounds_max = rounds_max;
        if (got) {
          if (RG == 5) {
            stk_item<5, 3>(ta, it, lane);
          } else if (RG == 4) {
            stk_item<4, 3>(ta, it, lane);
          } else {
            if (rr == 3) stk_item<2, 3>(ta, it, lane);
            else stk_item<2, 4>(ta, it, lane);
          }
        }
        __syncwarp();
        if (lane == 0) {
          const int nit = ((nr + RG - 1) / RG) * nrg;
          if (atomicAdd(&s_done[s], 1) == nit - 1) {
            atomicExch(&s_done[s], 0);
            mbar_arrive(&empty[s]);
          }
        }
      }
      seq += (uint32_t)(ph.ntl[0] + ph.ntl[1]);
    }
    stk_consumer_sync();
    // row results (round groups in order) back into red[mi][row][0]; a
    // matrix whose items span all rounds of a row has nothing to add
    bool more = false;
    for (int mi = 0; mi < ph.nm; ++mi) {
      const int nrg = ph.nrg[mi];
      if (nrg == 1) continue;
      more = true;
      for (int i = ctid; i < nrows; i += kStkConsThreads) {
        float *rw = red + ((size_t)mi * rows_max + i) * rounds_max;
        float sum = rw[0];
        for (int rd = 1; rd < nrg; ++rd) sum += rw[rd];
        rw[0] = sum;
      }
    }
    if (more) stk_consumer_sync();
  };

  // ---- prologue: t shares of layer 0's gate and up from x, entries [d_a, d_b)
  fetch_layer(0);
  if (p.L > 1) fetch_layer(1);
  stk_cp_async_wait_all();
  stk_consumer_sync();
  set_phase(0, 0, false);
  const StkPhase &ph = *sph;
  prefetch(ph, 0, kStkConsThreads);
  {
    const int n = d_b - d_a;
    for (int i = ctid; i < n; i += kStkConsThreads) vals[i] = bf16_bits_to_f32(p.x[d_a + i]);
    stk_consumer_sync();
    for (int j = 0; j < 2; ++j) {
      const StackMatDesc &m = ph.m[j];
      for (int k = cw; k < m.r; k += kStkCons) {
        const float *row = m.vh + (size_t)k * m.K + d_a;
        float sacc = 0.0f;
        for (int i = lane; i < n; i += 32) sacc = fmaf(__ldg(row + i), vals[i], sacc);
#pragma unroll
        for (int o = 16; o; o >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
        if (lane == 0) p.tp[((size_t)j * kStkMaxRank + k) * stk_gp(G) + c] = sacc;
      }
    }
  }
  grid_arrive();
  bool live = grid_wait();

  // ---- the blocks: gate+up (x -> h), then down (h -> x).  One loop over the
  // 2 L phases with a single call site per step, so that the phase's code
  // exists once in the kernel (it is executed once per phase and must stay
  // within the instruction caches).
  for (int step = 0; step < 2 * p.L; ++step) {
    const int l = step >> 1, kind = step & 1;
    // layer l + 1 into the slot of layer l - 1, whose last phase descriptor
    // was built at the previous barrier; it lands before this phase's rows
    if (kind == 0 && l >= 1 && l + 1 < p.L && live) fetch_layer(l + 1);
    if (live) run_phase(ph);
    if (kind == 0) {
      // h = RN_bf16(gelu(g) u), g and u rounded to BF16 first
      const int n = gu_b - gu_a;
      for (int i = ctid; i < n && live; i += kStkConsThreads) {
        const float gv = bf16_bits_to_f32(f32_to_bf16_rn_bits(red[(size_t)i * rounds_max]));
        const float uv =
            bf16_bits_to_f32(f32_to_bf16_rn_bits(red[((size_t)rows_max + i) * rounds_max]));
        const uint16_t hb = f32_to_bf16_rn_bits(gelu_erf(gv) * uv);
        p.h[gu_a + i] = hb;
        vals[i] = bf16_bits_to_f32(hb);
      }
    } else {
      const int n = d_b - d_a;
      for (int i = ctid; i < n && live; i += kStkConsThreads) {
        const uint16_t xb = f32_to_bf16_rn_bits(red[(size_t)i * rounds_max]);
        p.y[d_a + i] = xb;
        vals[i] = bf16_bits_to_f32(xb);
      }
    }
    stk_cp_async_wait_all();
    stk_consumer_sync();
    if (step + 1 == 2 * p.L) break;     // the last block's output needs no t shares
    if (live) t_share_out(ph);
    grid_arrive();
    // consumer warp 0 goes straight to the wait (its thread 0 polls); the
    // other warps build the next phase's descriptor and issue its prefetch
    if (cw >= 1) {
      set_phase(kind == 0 ? l : l + 1, kind ^ 1, true);
      prefetch(ph, 32, kStkPrepThreads);
    }
    live = grid_wait() && live;
  }
}

// --------------------------------------------------------------- host ---
namespace {
constexpr int kStkSlotTarget = 16384;      // bytes of weights per ring slot, about
constexpr int kStkSmemLimit = 232448;      // opt-in shared memory per CTA (227 KB)

int stk_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

int stk_row_bytes(const StackMatDesc &m) { return m.K / 2 + m.K / 32 + m.n_sal + 2 * m.r; }

struct StkWs {
  size_t desc, vh, tp, gbar, h, total;
};
StkWs stk_ws_layout(const StackShapeInfo &si, int L, int G) {
  StkWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  w.desc = take((size_t)L * sizeof(StackLayerDesc));
  w.vh = take(si.vh_floats * sizeof(float));
  w.tp = take((size_t)3 * kStkMaxRank * stk_gp(G) * sizeof(float));
  w.gbar = take(256);
  w.h = take((size_t)si.I * 2);
  w.total = off;
  return w;
}

bool stk_plan(const std::vector<StackLayerDesc> &Ls, int G, StackParams &p) {
  if (G < 1 || G > 32 * kStkShareRegs) return false;   // t shares a lane holds in registers
  const int L = (int)Ls.size();
  p.L = L;
  p.H = Ls[0].m[2].M;
  p.I = Ls[0].m[0].M;
  p.G = G;
  int rb_gu = 0, rb_d = 0, max_rank = 0, max_nsal = 0, rounds_max = 1;
  for (const auto &Ld : Ls)
    for (int mi = 0; mi < 3; ++mi) {
      const StackMatDesc &m = Ld.m[mi];
      if (mi < 2) rb_gu = std::max(rb_gu, stk_row_bytes(m));
      else rb_d = std::max(rb_d, stk_row_bytes(m));
      max_rank = std::max(max_rank, m.r);
      max_nsal = std::max(max_nsal, m.n_sal);
      rounds_max = std::max(rounds_max, (m.K / 32 + m.n_sal / 32 + 31) / 32);
    }
  p.tr_gu = std::max(2, (kStkSlotTarget / rb_gu) & ~1);
  // gate/up tiles of six rows or more grow to a multiple of ten: two
  // five-row items per tile (the Spark shapes: 8 -> 10 rows, 17.3 KB)
  if (p.tr_gu >= 6) p.tr_gu = (p.tr_gu + 9) / 10 * 10;
  p.tr_d = std::max(2, (kStkSlotTarget / rb_d) & ~1);
  p.slot_bytes = (std::max(p.tr_gu * rb_gu, p.tr_d * rb_d) + 127) & ~127;
  p.max_rank = max_rank;
  p.max_nsal = std::max(max_nsal, 32);
  p.rows_max = (std::max(p.H, p.I) + G - 1) / G + 1;
  p.rounds_max = rounds_max;
  const int Kmax = std::max(p.H, p.I);
  int off = 0;
  auto take = [&](int bytes) {
    const int o = off;
    off += (bytes + 127) & ~127;
    return o;
  };
  p.o_xi = take(Kmax * 2);
  p.o_xsc = take(Kmax / 64 * 4);
  p.o_xs8 = take(Kmax / 32 * 4);
  p.o_xs = take(2 * p.max_nsal * 2);
  p.o_xss = take(2 * (p.max_nsal / 32) * 4);
  p.o_sidx = take(2 * p.max_nsal * 4);
  p.o_t = take(2 * kStkMaxRank * 4);
  p.o_s8 = take(2 * stk_s8_stride(p.rows_max) * 2);
  p.o_yv = take(2 * p.rows_max * p.rounds_max * 4);
  p.o_vh = take(p.rows_max * 4);
  {
    const int rg = (p.I + G - 1) / G, rd = (p.H + G - 1) / G;
    p.o_vhs = take(std::max(max_rank * rg, 2 * max_rank * rd) * 4);
  }
  p.o_flag = take(16);
  p.o_grab = take((1 + 2 * kStkMaxSlots) * 4);
  p.o_ph = take((int)sizeof(StkPhase));
  p.o_ld = take(2 * (int)sizeof(StackLayerDesc));
  const int fixed = off;
  const int room = kStkSmemLimit - 1024 - fixed - 2 * kStkMaxSlots * 8 - 128;
  p.nslots = std::min(kStkMaxSlots, room / p.slot_bytes);
  if (p.nslots < 2) return false;
  p.o_full = take(p.nslots * 8);
  p.o_empty = take(p.nslots * 8);
  off = (off + 1023) & ~1023;
  p.o_ring = off;
  off += p.nslots * p.slot_bytes;
  p.smem_total = off + 1024;
  return p.smem_total <= kStkSmemLimit;
}
}  // namespace

bool stack_shape_info(const StackMatDesc *mats, int L, StackShapeInfo &si) {
  if (L < 1) return false;
  const int I = mats[0].M, H = mats[0].K, B = mats[0].block;
  if (H % 512 != 0 || I % 512 != 0) return false;
  size_t vh = 0;
  for (int l = 0; l < L; ++l)
    for (int mi = 0; mi < 3; ++mi) {
      const StackMatDesc &m = mats[3 * l + mi];
      const int M = mi < 2 ? I : H, K = mi < 2 ? H : I;
      if (m.M != M || m.K != K || m.block != B) return false;
      if (m.r < 0 || m.r > kStkMaxRank || m.r % 8 != 0) return false;
      if (m.n_sal % 32 != 0 || m.n_sal > K) return false;
      vh += (size_t)m.r * K;
    }
  si.H = H;
  si.I = I;
  si.block = B;
  si.vh_floats = vh;
  return true;
}

size_t stack_workspace_bytes(const StackShapeInfo &si, int L) {
  return stk_ws_layout(si, L, std::max(1, stk_sm_count())).total;
}

bool stack_plan_info(const StackMatDesc *mats, int L, int G, StackPlanInfo &out) {
  std::vector<StackLayerDesc> Ls((size_t)L);
  for (int l = 0; l < L; ++l)
    for (int mi = 0; mi < 3; ++mi) Ls[(size_t)l].m[mi] = mats[3 * l + mi];
  StackParams p{};
  if (!stk_plan(Ls, G, p)) return false;
  out.ctas = G;
  out.threads = kStkThreads;
  out.slots = p.nslots;
  out.slot_bytes = p.slot_bytes;
  out.tr_gu = p.tr_gu;
  out.tr_d = p.tr_d;
  out.smem = p.smem_total;
  return true;
}

cudaError_t stack_prepare(StackMatDesc *mats, int L, const StackShapeInfo &si, void *ws,
                          cudaStream_t st, Launcher &Lc) {
  const int G = stk_sm_count();
  if (G <= 0) return cudaErrorNoDevice;
  const StkWs w = stk_ws_layout(si, L, G);
  char *base = static_cast<char *>(ws);
  float *vh = reinterpret_cast<float *>(base + w.vh);
  std::vector<StackLayerDesc> Ls((size_t)L);
  for (int l = 0; l < L; ++l)
    for (int mi = 0; mi < 3; ++mi) {
      StackMatDesc m = mats[3 * l + mi];
      if (m.r > 0) {
        // (V H_K) row by row: the blockwise FWHT of each row of V (H is symmetric)
        cudaError_t e = launch_fwht(m.V, vh, m.r, m.K, m.block, st, Lc);
        if (e != cudaSuccess) return e;
        m.vh = vh;
        vh += (size_t)m.r * m.K;
      } else {
        m.vh = nullptr;
      }
      Ls[(size_t)l].m[mi] = m;
    }
  cudaError_t e = cudaMemcpyAsync(base + w.desc, Ls.data(), Ls.size() * sizeof(StackLayerDesc),
                                  cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);     // Ls is a host temporary
}

cudaError_t launch_mlp_stack(const StackMatDesc *mats, int L, const StackShapeInfo &si,
                             const void *x, void *y, void *ws, cudaStream_t st, Launcher &Lc) {
  const int G = stk_sm_count();
  if (G <= 0) return cudaErrorNoDevice;
  std::vector<StackLayerDesc> Ls((size_t)L);
  for (int l = 0; l < L; ++l)
    for (int mi = 0; mi < 3; ++mi) Ls[(size_t)l].m[mi] = mats[3 * l + mi];
  StackParams p{};
  if (!stk_plan(Ls, G, p)) return cudaErrorNotSupported;
  const StkWs w = stk_ws_layout(si, L, G);
  char *base = static_cast<char *>(ws);
  p.layers = reinterpret_cast<const StackLayerDesc *>(base + w.desc);
  p.x = static_cast<const uint16_t *>(x);
  p.y = static_cast<uint16_t *>(y);
  p.h = reinterpret_cast<uint16_t *>(base + w.h);
  p.tp = reinterpret_cast<float *>(base + w.tp);
  p.gbar = reinterpret_cast<unsigned int *>(base + w.gbar);
  cudaError_t e = cudaMemsetAsync(p.gbar, 0, sizeof(unsigned int), st);
  if (e != cudaSuccess) return e;
  if (si.block == 256)
    return Lc.launch_coop("mlp_stack", mlp_stack_kernel<256>, dim3(G), dim3(kStkThreads),
                          (size_t)p.smem_total, st, p);
  return Lc.launch_coop("mlp_stack", mlp_stack_kernel<128>, dim3(G), dim3(kStkThreads),
                        (size_t)p.smem_total, st, p);
}

cudaError_t prepare_stack_kernels() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(mlp_stack_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kStkSmemLimit)) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(mlp_stack_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kStkSmemLimit);
}

}  // namespace dvssq
