// Dense effective weights from the packed form (Spark-X2.5-4B-Hadamard-GSQ
// model card, "Quickstart & Inference Guide": model.materialize_weights()
// turns the quantised MLP weights back into plain BF16):
//
//     W_eff = RN_bf16( (What4 + scatter(What8) + U V) . H_K )
//
// in the original, unrotated domain.  H_K = diag(H_b, ...) is symmetric and
// orthogonal, so W_eff x = (What4 + What8 + U V) (H_K x): the dense matrix
// gives the forward's result (MiniCPM5-2B-Hadamard-GSQ card, Mathematical
// Foundations §1, rotation invariance; §2, What = Q s and A B = U V).
//
// HBM-bound: per weight it reads half a byte of codes (plus scales, the INT8
// tier and U) and writes two bytes of BF16.  One warp owns a tile of 8 rows
// x one Hadamard block of b columns:
//   * the tile's codes, scales, U rows and INT8 entries arrive by cp.async
//     into a per-warp double buffer (the next tile's while this one runs);
//   * the FP32 accumulators start as q s4 (+ q8 s8 at salient columns) and
//     the rank-r term U V is added on the tensor cores (mma.sync m16n8k16,
//     BF16 operands, FP32 accumulation; U rows 0..7 of the A operand, V of
//     the block staged transposed in shared memory once per CTA and block);
//   * the b-point Walsh-Hadamard transform runs along the columns: the
//     accumulator of lane (g, q) holds row g's columns 8t + 2q + e, so the
//     butterflies over e and t stay in registers and the two over q are quad
//     shuffles; then the 1/sqrt(b) scale, BF16 rounding and 4-byte stores.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace dvssq {

constexpr int kMatWarps = 4;
constexpr int kMatThreads = 32 * kMatWarps;
constexpr int kMatRows = 8;                         // rows per warp tile
constexpr int kMatRowsCta = kMatRows * kMatWarps;   // rows per CTA item
constexpr int kMatMaxRank = 64;
constexpr int kMatURow = kMatMaxRank * 2 + 16;      // U bytes per staged row (padded)

// Packed FP32x2 arithmetic (sm_100a): two independent round-to-nearest
// operations per instruction.
__device__ __forceinline__ unsigned long long mat_f2u(float2 a) {
  return (unsigned long long)__float_as_uint(a.x) | ((unsigned long long)__float_as_uint(a.y) << 32);
}
__device__ __forceinline__ float2 mat_u2f(unsigned long long u) {
  return make_float2(__uint_as_float((uint32_t)u), __uint_as_float((uint32_t)(u >> 32)));
}
__device__ __forceinline__ float2 mat_add2(float2 a, float2 b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(mat_f2u(a)), "l"(mat_f2u(b)));
  return mat_u2f(r);
}
__device__ __forceinline__ float2 mat_sub2(float2 a, float2 b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(mat_f2u(a)), "l"(mat_f2u(b)));
  return mat_u2f(r);
}
__device__ __forceinline__ float2 mat_mul2(float2 a, float2 b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(mat_f2u(a)), "l"(mat_f2u(b)));
  return mat_u2f(r);
}
__device__ __forceinline__ float2 mat_fma2(float2 a, float2 b, float2 c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(mat_f2u(a)), "l"(mat_f2u(b)), "l"(mat_f2u(c)));
  return mat_u2f(r);
}

__device__ __forceinline__ void mat_cp_async(void *smem, const void *gmem, int bytes) {
  if (bytes == 16)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
  else if (bytes == 8)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
}
// 4-byte copy that reads only `src_bytes` (2 or 4) and zero-fills the rest
__device__ __forceinline__ void mat_cp_async4_zfill(void *smem, const void *gmem, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void mat_cp_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void mat_cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct MatParams {
  const uint8_t *q4;
  const uint16_t *s4;
  const int32_t *sal_idx;
  const int8_t *q8;
  const uint16_t *s8;
  const uint16_t *U;
  const uint16_t *V;
  uint16_t *W;            // BF16 [M][K]
  int M, K, n_sal, r, rp; // rp: rank rounded up to 16
  int nrt;                // CTA row items per column block
  long long nitems;       // nkb * nrt
  float c;                // 1/sqrt(b) in FP32
};

// Per-warp stage layout (bytes from the stage base).
template <int B>
struct MatStage {
  static constexpr int kQ4Row = B / 2 + 16;         // padded: the 8 rows hit distinct banks
  static constexpr int kQ8Row = B + 16;             // salient entries of one block, 16-B chunks
  static constexpr int q4 = 0;
  static constexpr int s4 = q4 + kMatRows * kQ4Row;
  static constexpr int s8 = s4 + kMatRows * 8;
  static constexpr int u = s8 + kMatRows * 4;
  static constexpr int q8 = u + kMatRows * kMatURow;
  static constexpr int bytes = (q8 + kMatRows * kQ8Row + 15) & ~15;
};

template <int B>
__global__ void __launch_bounds__(kMatThreads, 3) materialize_kernel(const MatParams p) {
  constexpr int NT = B / 8;                  // n-tiles of 8 columns
  using St = MatStage<B>;
  extern __shared__ __align__(16) unsigned char mat_smem[];
  const int nkb = p.K / B;
  const int vtw = p.rp / 2 + 4;              // 32-bit words per column of the staged V^T
  // layout: [stages: kMatWarps x 2 x St::bytes][V^T: B x vtw words]
  //         [V rows: r x (B + 8) BF16][tab: B int16][pref: nkb + 1]
  unsigned char *stages = mat_smem;
  uint32_t *vt = reinterpret_cast<uint32_t *>(mat_smem + kMatWarps * 2 * St::bytes);
  uint16_t *vrm = reinterpret_cast<uint16_t *>(vt + B * vtw);
  int16_t *tab = reinterpret_cast<int16_t *>(vrm + p.rp * (B + 8));
  int *pref = reinterpret_cast<int *>(tab + B);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;

  // first salient slot of every column block (sal_idx is ascending)
  for (int k = tid; k <= nkb; k += kMatThreads) {
    const int key = k * B;
    int lo = 0, hi = p.n_sal;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (p.sal_idx[mid] < key) lo = mid + 1;
      else hi = mid;
    }
    pref[k] = lo;
  }
  __syncthreads();

  const long long per = (p.nitems + gridDim.x - 1) / gridDim.x;
  const long long i0 = (long long)blockIdx.x * per;
  const long long i1 = min(p.nitems, i0 + per);
  if (i0 >= i1) return;

  // stage the warp's tile of item `it` into buffer `buf`
  auto prefetch = [&](long long it, int buf) {
    const int kb = (int)(it / p.nrt), rt = (int)(it - (long long)kb * p.nrt);
    unsigned char *st = stages + (warp * 2 + buf) * St::bytes;
    const int rr = lane >> 2, sub = lane & 3;           // 4 lanes per row
    const int row = rt * kMatRowsCta + warp * kMatRows + rr;
    if (row < p.M) {
      const unsigned char *q4r = p.q4 + (size_t)row * (p.K / 2) + (size_t)kb * (B / 2);
      for (int c = sub; c < B / 32; c += 4)
        mat_cp_async(st + St::q4 + rr * St::kQ4Row + 16 * c, q4r + 16 * c, 16);
      if (sub == 0) {
        mat_cp_async(st + St::s4 + rr * 8, p.s4 + (size_t)row * (p.K / 64) + (size_t)kb * (B / 64),
                     B / 32);
        // the aligned pair holding s8[row]; the last row of an odd M reads
        // only its own two bytes
        mat_cp_async4_zfill(st + St::s8 + rr * 4, p.s8 + (row & ~1), (row | 1) < p.M ? 4 : 2);
      }
      if (p.r > 0)
        for (int c = sub; c < p.r / 8; c += 4)
          mat_cp_async(st + St::u + rr * kMatURow + 16 * c, p.U + (size_t)row * p.r + 8 * c, 16);
      const int cs = pref[kb] & ~15, ce = (pref[kb + 1] + 15) & ~15;
      for (int c = cs + 16 * sub; c < ce; c += 64)
        mat_cp_async(st + St::q8 + rr * St::kQ8Row + (c - cs), p.q8 + (size_t)row * p.n_sal + c, 16);
    }
    mat_cp_commit();
  };

  int cur_kb = -1;
  prefetch(i0, 0);
  int buf = 0;
  for (long long it = i0; it < i1; ++it, buf ^= 1) {
    const int kb = (int)(it / p.nrt), rt = (int)(it - (long long)kb * p.nrt);
    if (kb != cur_kb) {
      // V of this column block: its rows by cp.async (all copies in flight
      // at once) into the row-major staging area, then transposed in shared
      // memory into column-major BF16 pairs; and the salient slot of every
      // column of the block
      __syncthreads();
      for (int i = tid; i < p.r * (B / 8); i += kMatThreads) {
        const int rho = i / (B / 8), c = i - rho * (B / 8);
        mat_cp_async(vrm + rho * (B + 8) + 8 * c, p.V + (size_t)rho * p.K + (size_t)kb * B + 8 * c,
                     16);
      }
      mat_cp_commit();
      for (int i = tid; i < B; i += kMatThreads) tab[i] = -1;
      mat_cp_wait<0>();
      __syncthreads();
      for (int e = pref[kb] + tid; e < pref[kb + 1]; e += kMatThreads)
        tab[p.sal_idx[e] - kb * B] = (int16_t)e;
      for (int i = tid; i < B * (p.rp / 2); i += kMatThreads) {
        const int col = i % B, pr = i / B;            // rank pair (2 pr, 2 pr + 1)
        const uint32_t lo = 2 * pr < p.r ? vrm[(2 * pr) * (B + 8) + col] : 0u;
        const uint32_t hi = 2 * pr + 1 < p.r ? vrm[(2 * pr + 1) * (B + 8) + col] : 0u;
        vt[col * vtw + pr] = lo | (hi << 16);
      }
      __syncthreads();
      cur_kb = kb;
    }
    if (it + 1 < i1) {
      prefetch(it + 1, buf ^ 1);
      mat_cp_wait<1>();
    } else {
      mat_cp_wait<0>();
    }
    __syncwarp();
    const unsigned char *st = stages + (warp * 2 + buf) * St::bytes;
    const int row = rt * kMatRowsCta + warp * kMatRows + g;

    // accumulators: column 8t + 2q + e of row g
    float acc[NT][2];
    {
      const uint2 sw = *reinterpret_cast<const uint2 *>(st + St::s4 + g * 8);
      float s4f[4];
      s4f[0] = bf16_bits_to_f32(sw.x & 0xFFFFu);
      s4f[1] = bf16_bits_to_f32(sw.x >> 16);
      s4f[2] = bf16_bits_to_f32(sw.y & 0xFFFFu);
      s4f[3] = bf16_bits_to_f32(sw.y >> 16);
      const unsigned char *qrow = st + St::q4 + g * St::kQ4Row;
#pragma unroll
      for (int t4 = 0; t4 < NT / 4; ++t4) {
        const uint4 w = *reinterpret_cast<const uint4 *>(qrow + 16 * t4);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int t = 4 * t4 + k;
          const uint32_t byte = (ww[k] >> (8 * q)) & 0xFFu;
          const int lo = (int)(byte << 28) >> 28, hi = (int)(byte << 24) >> 28;
          const float s = s4f[t >> 3];
          acc[t][0] = (float)lo * s;
          acc[t][1] = (float)hi * s;
        }
      }
    }
    // the INT8 tier, scattered to its columns
    if (pref[kb + 1] > pref[kb]) {
      const uint32_t s8w = *reinterpret_cast<const uint32_t *>(st + St::s8 + g * 4);
      const float s8f = bf16_bits_to_f32((row & 1) ? (s8w >> 16) : (s8w & 0xFFFFu));
      const int cs = pref[kb] & ~15;
      const signed char *q8r =
          reinterpret_cast<const signed char *>(st + St::q8 + g * St::kQ8Row) - cs;
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int slot = tab[8 * t + 2 * q + e];
          if (slot >= 0) acc[t][e] += (float)q8r[slot] * s8f;
        }
    }
    // + U V on the tensor cores (A rows 8..15 are zero)
    if (p.r > 0) {
      const unsigned char *urow = st + St::u + g * kMatURow;
      for (int ks = 0; ks < p.rp / 16; ++ks) {
        const int k0 = 16 * ks + 2 * q, k1 = k0 + 8;
        uint32_t a[4];
        a[0] = k0 < p.r ? *reinterpret_cast<const uint32_t *>(urow + 2 * k0) : 0u;
        a[1] = 0u;
        a[2] = k1 < p.r ? *reinterpret_cast<const uint32_t *>(urow + 2 * k1) : 0u;
        a[3] = 0u;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint32_t *vc = vt + (8 * t + g) * vtw + 8 * ks + q;
          float d[4] = {acc[t][0], acc[t][1], 0.f, 0.f};
          mma_bf16_16816(d, a, vc[0], vc[4]);
          acc[t][0] = d[0];
          acc[t][1] = d[1];
        }
      }
    }
    // Walsh-Hadamard transform along the b columns: bit 0 (e) and bits 3..
    // (t) in registers, bits 1 and 2 (q) across the quad.  After the e stage
    // the (e = 0, 1) pair of every t runs as one packed FP32x2 operation; a
    // quad stage is o + (+-1) v by one packed FMA (v times +-1 is exact, so
    // the single rounding equals that of the scalar add or subtract).
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float a0 = acc[t][0], a1 = acc[t][1];
      acc[t][0] = a0 + a1;
      acc[t][1] = a0 - a1;
    }
    float2 v[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) v[t] = make_float2(acc[t][0], acc[t][1]);
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
      const float sg = (q & m) ? -1.0f : 1.0f;
      const float2 sg2 = make_float2(sg, sg);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float2 o;
        o.x = __shfl_xor_sync(0xffffffffu, v[t].x, m);
        o.y = __shfl_xor_sync(0xffffffffu, v[t].y, m);
        v[t] = mat_fma2(v[t], sg2, o);
      }
    }
#pragma unroll
    for (int h = 1; h < NT; h <<= 1)
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (!(t & h)) {
          const float2 a0 = v[t], a1 = v[t + h];
          v[t] = mat_add2(a0, a1);
          v[t + h] = mat_sub2(a0, a1);
        }
    if (row < p.M) {
      uint32_t *dst = reinterpret_cast<uint32_t *>(p.W + (size_t)row * p.K + (size_t)kb * B) + q;
      const float2 c2 = make_float2(p.c, p.c);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float2 w = mat_mul2(v[t], c2);
        const __nv_bfloat162 hb = __floats2bfloat162_rn(w.x, w.y);   // .x in the low half
        dst[4 * t] = *reinterpret_cast<const uint32_t *>(&hb);
      }
    }
    __syncwarp();
  }
}

namespace {
size_t mat_smem_bytes(int B, int rp) {
  const size_t st = B == 256 ? MatStage<256>::bytes : MatStage<128>::bytes;
  return kMatWarps * 2 * st + (size_t)B * (rp / 2 + 4) * 4 + (size_t)rp * (B + 8) * 2 +
         (size_t)B * 2 + (size_t)(65536 / 128 + 1) * 4;
}
}  // namespace

cudaError_t launch_materialize(const MaterializeArgs &a, cudaStream_t st, Launcher &L) {
  MatParams p{};
  p.q4 = a.q4; p.s4 = a.s4; p.sal_idx = a.sal_idx; p.q8 = a.q8; p.s8 = a.s8;
  p.U = a.U; p.V = a.V; p.W = a.W;
  p.M = a.M; p.K = a.K; p.n_sal = a.n_sal; p.r = a.rank;
  p.rp = (a.rank + 15) / 16 * 16;
  p.nrt = (a.M + kMatRowsCta - 1) / kMatRowsCta;
  p.nitems = (long long)(a.K / a.block) * p.nrt;
  p.c = (float)(1.0 / sqrt((double)a.block));
  const size_t smem = mat_smem_bytes(a.block, p.rp);
  int dev = 0, nsm = 0, occ = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  auto kern = a.block == 256 ? materialize_kernel<256> : materialize_kernel<128>;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kMatThreads, smem)) !=
      cudaSuccess)
    return e;
  const long long grid = std::max(1LL, std::min<long long>(p.nitems, (long long)nsm * std::max(1, occ)));
  return L.launch("materialize", kern, dim3((unsigned)grid), dim3(kMatThreads), smem, st, false, p);
}

cudaError_t prepare_materialize_kernels() {
  cudaError_t e;
  for (const void *f : {(const void *)materialize_kernel<256>, (const void *)materialize_kernel<128>})
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)mat_smem_bytes(256, kMatMaxRank))) != cudaSuccess)
      return e;
  return cudaSuccess;
}

}  // namespace dvssq
