// Truncated SVD of the INT4 residual on the GPU (Spark-X2.5-4B-Hadamard-GSQ
// model card, Tier C, "Truncated SVD Low-Rank Residual Compensation":
// R = W_bg - What_bg ~= U_r S_r V_r^T; MiniCPM5-2B-Hadamard-GSQ card,
// Mathematical Foundations §2: A = U_r sqrt(S_r), B = sqrt(S_r) V_r^T), by
// randomised subspace iteration:
//
//   Y = R X (X: K x p Gaussian, p = r + 16)        Q = orth(Y)
//   q times:  Z = orth(R^T Q),  Q = orth(R Z)
//   Bt = R^T Q (K x p),  G = Bt^T Bt = W diag(lambda) W^T  (p x p, Jacobi)
//   A = Q W_r diag(lambda_r^(1/4)),  B = diag(lambda_r^(-1/4)) W_r^T Bt^T
//
// so that A B = Q Q^T R projected on the leading r eigenvectors of G: the
// rank-r truncation of R within the subspace range(Q), which approaches the
// Eckart-Young optimum as q grows.  orth() is shifted CholeskyQR applied
// twice (Gram matrix in fp64, Cholesky and triangular inverse in fp64 in one
// CTA); the products with R are FP32 on the CUDA cores, the eigenproblem
// fp64.  Every reduction runs in a fixed order: results are deterministic.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>
#include <cmath>

namespace dvssq {

constexpr int kLrOver = 16;          // oversampling p - r
constexpr int kLrMaxP = 80;          // rank <= 64
constexpr int kLrTile = 128;         // outputs (rows or columns of R) per CTA in the products
constexpr int kLrSlice = 512;        // longest inner-dimension slice per CTA in the products
constexpr int kLrMinSlice = 128;     // shortest
constexpr int kLrChunk = 32;         // inner-dimension chunk staged in shared memory
constexpr int kLrThreads = 256;
constexpr int kLrGramRows = 128;     // rows per partial Gram matrix

// Counter-based standard normal numbers: splitmix64 of (seed, index) gives
// two uniforms, Box-Muller turns them into one N(0, 1) value.
__device__ __forceinline__ uint64_t lr_mix(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void lr_gaussian_kernel(float *X, long long n, uint64_t seed) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const uint64_t a = lr_mix(seed ^ lr_mix((uint64_t)(2 * i))), b = lr_mix(seed ^ lr_mix((uint64_t)(2 * i + 1)));
    const double u1 = ((double)(a >> 11) + 0.5) * 0x1p-53, u2 = (double)(b >> 11) * 0x1p-53;
    X[i] = (float)(sqrt(-2.0 * log(u1)) * cospi(2.0 * u2));
  }
}

// Split products with R, FP32 on the CUDA cores.  A CTA owns a tile of 128
// outputs (rows of R for R X, columns of R for R^T Q) x all p columns, over
// one slice (a multiple of kLrChunk) along the inner dimension; thread (og, cg) = (tid / 8,
// tid % 8) accumulates outputs 4 og .. 4 og + 3 x columns p/8 cg .. (register
// blocking: one 16-byte load of R and p/8 values of the small operand feed
// p/2 FMAs per step, and a warp's loads of a step are two shared-memory
// wavefronts for 16 p FMAs).  The next chunk of R and of the small operand is
// loaded into registers while the current chunk runs from shared memory.
// Partial results go to part[slice][n][p], summed in slice order by
// lr_reduce_kernel.
//   TRANS = 0: out[i][j] = sum_k R[i][k] X[k][j]   (n = M, inner = K)
//   TRANS = 1: out[c][j] = sum_i R[i][c] Q[i][j]   (n = K, inner = M)
template <int P, int TRANS>
__global__ void __launch_bounds__(kLrThreads) lr_mul_kernel(const float *__restrict__ R,
                                                            const float *__restrict__ B,
                                                            float *__restrict__ part, int M,
                                                            int K, int slice) {
  constexpr int PG = P / 8;                      // columns per thread
  static_assert(kLrThreads == 8 * (kLrTile / 4), "8 column groups x kLrTile / 4 output groups");
  constexpr int RE = kLrChunk * kLrTile / kLrThreads;   // R values per thread and chunk (16)
  constexpr int XE = kLrChunk * P / kLrThreads;  // small-operand values per thread and chunk
  constexpr int RS = kLrTile + 8;                // padded row of the staged R chunk
  __shared__ __align__(16) float rs[kLrChunk][RS];      // [inner][out]
  __shared__ __align__(16) float bs[kLrChunk][P];
  const int tid = threadIdx.x, og = tid >> 3, cg = tid & 7;
  const int n = TRANS ? K : M, inner = TRANS ? M : K;
  const int o0 = blockIdx.x * kLrTile;
  const int t0 = blockIdx.y * slice, t1 = min(inner, t0 + slice);
  float acc[4][PG];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int j = 0; j < PG; ++j) acc[a][j] = 0.f;
  float rr[RE], br[XE];
  auto load = [&](int c0) {
#pragma unroll
    for (int u = 0; u < RE; ++u) {
      const int e = tid + u * kLrThreads;
      int o, t;
      if (TRANS) { t = e / kLrTile; o = e % kLrTile; }   // consecutive threads: consecutive columns
      else { o = e / kLrChunk; t = e % kLrChunk; }       // consecutive threads: consecutive k
      const int go = o0 + o, gt = c0 + t;
      rr[u] = (go < n && gt < t1) ? (TRANS ? R[(size_t)gt * K + go] : R[(size_t)go * K + gt]) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < XE; ++u) {
      const int e = tid + u * kLrThreads, t = e / P, j = e - t * P;
      br[u] = c0 + t < t1 ? B[(size_t)(c0 + t) * P + j] : 0.f;
    }
  };
  auto store = [&]() {
#pragma unroll
    for (int u = 0; u < RE; ++u) {
      const int e = tid + u * kLrThreads;
      if (TRANS) rs[e / kLrTile][e % kLrTile] = rr[u];
      else rs[e % kLrChunk][e / kLrChunk] = rr[u];
    }
#pragma unroll
    for (int u = 0; u < XE; ++u) {
      const int e = tid + u * kLrThreads;
      bs[e / P][e % P] = br[u];
    }
  };
  load(t0);
  for (int c0 = t0; c0 < t1; c0 += kLrChunk) {
    __syncthreads();
    store();
    __syncthreads();
    if (c0 + kLrChunk < t1) load(c0 + kLrChunk);
#pragma unroll 4
    for (int t = 0; t < kLrChunk; ++t) {
      const float4 ra = *reinterpret_cast<const float4 *>(&rs[t][4 * og]);
      const float rv[4] = {ra.x, ra.y, ra.z, ra.w};
      float bv[PG];
      if constexpr (PG % 4 == 0) {
#pragma unroll
        for (int j = 0; j < PG; j += 4) {
          const float4 b4 = *reinterpret_cast<const float4 *>(&bs[t][cg * PG + j]);
          bv[j] = b4.x; bv[j + 1] = b4.y; bv[j + 2] = b4.z; bv[j + 3] = b4.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < PG; j += 2) {
          const float2 b2 = *reinterpret_cast<const float2 *>(&bs[t][cg * PG + j]);
          bv[j] = b2.x; bv[j + 1] = b2.y;
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int j = 0; j < PG; ++j) acc[a][j] = fmaf(rv[a], bv[j], acc[a][j]);
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
    if (o0 + 4 * og + a < n)
#pragma unroll
      for (int j = 0; j < PG; ++j)
        part[((size_t)blockIdx.y * n + o0 + 4 * og + a) * P + cg * PG + j] = acc[a][j];
}

// out[n][p] = sum over slices of part[slice][n][p], in slice order.
__global__ void lr_reduce_kernel(const float *__restrict__ part, int nslices, long long count,
                                 float *__restrict__ out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (long long)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int sl = 0; sl < nslices; ++sl) s += part[(size_t)sl * count + i];
    out[i] = s;
  }
}

// Partial Gram matrices in fp64: part[b] = Y[rows of block b]^T Y[...] over
// kLrGramRows rows, staged 128 at a time (sub-chunks summed in order).
template <int P>
__global__ void __launch_bounds__(kLrThreads) lr_gram_kernel(const float *__restrict__ Y, int n,
                                                             double *__restrict__ part) {
  constexpr int SUB = 128;
  constexpr int EPT = (P * P + kLrThreads - 1) / kLrThreads;   // entries per thread
  constexpr int LPT = SUB * P / kLrThreads;                     // staged values per thread
  __shared__ float ys[SUB][P];
  const int r0 = blockIdx.x * kLrGramRows;
  double acc[EPT];
#pragma unroll
  for (int u = 0; u < EPT; ++u) acc[u] = 0.0;
  for (int s0 = 0; s0 < kLrGramRows; s0 += SUB) {
    float v[LPT];
#pragma unroll
    for (int u = 0; u < LPT; ++u) {
      const int i = threadIdx.x + u * kLrThreads, rr = i / P;
      v[u] = r0 + s0 + rr < n ? Y[(size_t)(r0 + s0) * P + i] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < LPT; ++u) {
      const int i = threadIdx.x + u * kLrThreads;
      ys[i / P][i % P] = v[u];
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < EPT; ++u) {
      const int e = threadIdx.x + u * kLrThreads;
      if (e < P * P) {
        const int a = e / P, b = e - a * P;
        double s = acc[u];
        for (int rr = 0; rr < SUB; ++rr) s = fma((double)ys[rr][a], (double)ys[rr][b], s);
        acc[u] = s;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < EPT; ++u) {
    const int e = threadIdx.x + u * kLrThreads;
    if (e < P * P) part[(size_t)blockIdx.x * P * P + e] = acc[u];
  }
}

// sum_b part[b * stride + e] in ascending b; the loads of a batch are issued
// together, the adds keep their order
__device__ __forceinline__ double lr_sum_parts(const double *__restrict__ part, int nparts, int e,
                                               int stride) {
  double s = 0.0;
  for (int b0 = 0; b0 < nparts; b0 += 16) {
    double v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = b0 + u < nparts ? part[(size_t)(b0 + u) * stride + e] : 0.0;
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (b0 + u < nparts) s += v[u];
  }
  return s;
}

// M[a][b] (row stride P + 1) = sum_b part[b][a][b] in ascending b for all
// P x P entries: each thread's entries with a batch of partials each in
// flight together (32 loads at most), the adds in order.
template <int P, int NT = kLrThreads>
__device__ __forceinline__ void lr_fill_sums(const double *__restrict__ part, int nparts,
                                             double *M) {
  constexpr int EPT = (P * P + NT - 1) / NT;
  constexpr int KB = EPT >= 32 ? 1 : 32 / EPT;      // partials per batch: <= 32 loads in flight
  double acc[EPT];
#pragma unroll
  for (int u = 0; u < EPT; ++u) acc[u] = 0.0;
  for (int b0 = 0; b0 < nparts; b0 += KB) {
    double v[EPT][KB];
#pragma unroll
    for (int u = 0; u < EPT; ++u) {
      const int e = threadIdx.x + u * NT;
#pragma unroll
      for (int k = 0; k < KB; ++k)
        v[u][k] = (e < P * P && b0 + k < nparts) ? part[(size_t)(b0 + k) * P * P + e] : 0.0;
    }
#pragma unroll
    for (int u = 0; u < EPT; ++u)
#pragma unroll
      for (int k = 0; k < KB; ++k)
        if (b0 + k < nparts) acc[u] += v[u][k];
  }
#pragma unroll
  for (int u = 0; u < EPT; ++u) {
    const int e = threadIdx.x + u * NT;
    if (e < P * P) M[(e / P) * (P + 1) + e % P] = acc[u];
  }
}

// One CTA: G = sum of the partials (in block order), shifted Cholesky
// G + s I = L L^T with s = 1e-12 trace(G), right-looking: column j of L and
// the rank-one update of the trailing matrix by all threads, one barrier per
// column (each entry's updates keep the column order of a left-looking
// factorisation).  A zero block (trace 0) writes L = 0, which the solve
// maps to zero rows.
constexpr int kLrCholThreads = 512;
template <int P>
__global__ void __launch_bounds__(kLrCholThreads) lr_chol_kernel(const double *__restrict__ part,
                                                                 int nparts, double *__restrict__ Lout) {
  extern __shared__ double lr_dyn[];
  double(*A)[P + 1] = reinterpret_cast<double(*)[P + 1]>(lr_dyn);            // G + s I, updated
  double(*Lm)[P + 1] = reinterpret_cast<double(*)[P + 1]>(lr_dyn + P * (P + 1));
  __shared__ double s_shift;
  const int tid = threadIdx.x;
  lr_fill_sums<P, kLrCholThreads>(part, nparts, &A[0][0]);
  for (int e = tid; e < P * P; e += kLrCholThreads) Lm[e / P][e % P] = 0.0;
  __syncthreads();
  if (tid == 0) {
    double tr = 0.0;
    for (int j = 0; j < P; ++j) tr += A[j][j];
    s_shift = 1e-12 * tr;
  }
  __syncthreads();
  const double sh = s_shift;
  if (sh == 0.0) {
    for (int e = tid; e < P * P; e += kLrCholThreads) Lout[e] = 0.0;
    return;
  }
  if (tid < P) A[tid][tid] += sh;
  __syncthreads();
  for (int j = 0; j < P; ++j) {
    const double ljj = sqrt(fmax(A[j][j], sh));
    const int nc = P - 1 - j;                    // rows below j
    for (int e = tid; e < nc * (nc + 1); e += kLrCholThreads) {
      const int i = j + 1 + e / (nc + 1), k = j + e % (nc + 1);   // k = j: the column itself
      if (k > i) continue;
      const double lij = A[i][j] / ljj;
      if (k == j) {
        Lm[i][j] = lij;
      } else {
        const double lkj = A[k][j] / ljj;
        A[i][k] -= lij * lkj;
      }
    }
    if (tid == 0) Lm[j][j] = ljj;
    __syncthreads();
  }
  for (int e = tid; e < P * P; e += kLrCholThreads) Lout[e] = Lm[e / P][e % P];
}

// Y[n][p] <- Y L^-T (row y -> L^-1 y), in place, by forward substitution:
// one thread per row, the row in registers, L in shared memory (FP32, its
// reciprocal diagonal from fp64).  The dependency chain of a row is long
// but the rows run side by side.
constexpr int kLrSolveThreads = 64;
template <int P>
__global__ void __launch_bounds__(kLrSolveThreads) lr_apply_solve_kernel(float *__restrict__ Y, int n,
                                                                         const double *__restrict__ Lg) {
  __shared__ float Ls[P][P + 1];
  __shared__ float dinv[P];
  for (int e = threadIdx.x; e < P * P; e += kLrSolveThreads) Ls[e / P][e % P] = (float)Lg[e];
  for (int i = threadIdx.x; i < P; i += kLrSolveThreads) {
    const double d = Lg[i * P + i];
    dinv[i] = d != 0.0 ? (float)(1.0 / d) : 0.f;
  }
  __syncthreads();
  const long long r = (long long)blockIdx.x * kLrSolveThreads + threadIdx.x;
  if (r >= n) return;
  float4 *row = reinterpret_cast<float4 *>(Y + r * P);
  float y[P];
#pragma unroll
  for (int q = 0; q < P / 4; ++q) {
    const float4 v = row[q];
    y[4 * q] = v.x; y[4 * q + 1] = v.y; y[4 * q + 2] = v.z; y[4 * q + 3] = v.w;
  }
  // two partial sums per output halve the dependency chain
#pragma unroll
  for (int i = 0; i < P; ++i) {
    float s0 = y[i], s1 = 0.f;
#pragma unroll
    for (int k = 0; k + 1 < i; k += 2) {
      s0 = fmaf(-Ls[i][k], y[k], s0);
      s1 = fmaf(-Ls[i][k + 1], y[k + 1], s1);
    }
    if (i & 1) s0 = fmaf(-Ls[i][i - 1], y[i - 1], s0);
    y[i] = (s0 + s1) * dinv[i];
  }
#pragma unroll
  for (int q = 0; q < P / 4; ++q) row[q] = make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
}

// One CTA: eigen-decomposition of the symmetric G (sum of the partials) by
// cyclic Jacobi rotations, P/2 disjoint pairs per step in the round-robin
// order, sweeps until the off-diagonal mass is negligible.  Outputs the
// eigenvectors W (columns) and eigenvalues lam, sorted descending.
template <int P>
__global__ void __launch_bounds__(kLrThreads) lr_eig_kernel(const double *__restrict__ part,
                                                            int nparts, double *__restrict__ Wout,
                                                            double *__restrict__ lam_out) {
  extern __shared__ double lr_dyn[];
  double(*A)[P + 1] = reinterpret_cast<double(*)[P + 1]>(lr_dyn);
  double(*W)[P + 1] = reinterpret_cast<double(*)[P + 1]>(lr_dyn + P * (P + 1));
  __shared__ double cs[P / 2], sn[P / 2];
  __shared__ int pa[P / 2], pb[P / 2];
  __shared__ int perm[P];
  __shared__ double rowoff[P], rowdia[P];
  __shared__ double s_off;
  const int tid = threadIdx.x;
  lr_fill_sums<P>(part, nparts, &A[0][0]);
  for (int e = tid; e < P * P; e += kLrThreads) W[e / P][e % P] = (e / P == e % P) ? 1.0 : 0.0;
  if (tid < P) perm[tid] = tid;
  __syncthreads();
  for (int sweep = 0; sweep < 30; ++sweep) {
    // converged when the off-diagonal mass is below 1e-26 of the diagonal's
    // (rows summed by P threads, then by one)
    if (tid < P) {
      double off = 0.0, dia = 0.0;
      for (int j = 0; j < P; ++j) (tid == j ? dia : off) += A[tid][j] * A[tid][j];
      rowoff[tid] = off;
      rowdia[tid] = dia;
    }
    __syncthreads();
    if (tid == 0) {
      double off = 0.0, dia = 0.0;
      for (int i = 0; i < P; ++i) { off += rowoff[i]; dia += rowdia[i]; }
      s_off = off <= 1e-26 * dia ? 1.0 : 0.0;
    }
    __syncthreads();
    if (s_off != 0.0) break;
    for (int step = 0; step < P - 1; ++step) {
      // round-robin pairs: perm[k] with perm[P-1-k]
      if (tid < P / 2) {
        int a = perm[tid], b = perm[P - 1 - tid];
        if (a > b) { const int t = a; a = b; b = t; }
        pa[tid] = a;
        pb[tid] = b;
        const double apq = A[a][b];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double theta = (A[b][b] - A[a][a]) / (2.0 * apq);
          const double t = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
          c = 1.0 / sqrt(t * t + 1.0);
          s = t * c;
        }
        cs[tid] = c;
        sn[tid] = s;
      }
      __syncthreads();
      // rows: A <- J^T A
      for (int e = tid; e < (P / 2) * P; e += kLrThreads) {
        const int k = e / P, col = e - k * P;
        const int a = pa[k], b = pb[k];
        const double c = cs[k], s = sn[k];
        const double xa = A[a][col], xb = A[b][col];
        A[a][col] = c * xa - s * xb;
        A[b][col] = s * xa + c * xb;
      }
      __syncthreads();
      // columns: A <- A J, W <- W J
      for (int e = tid; e < (P / 2) * P; e += kLrThreads) {
        const int k = e / P, row = e - k * P;
        const int a = pa[k], b = pb[k];
        const double c = cs[k], s = sn[k];
        const double xa = A[row][a], xb = A[row][b];
        A[row][a] = c * xa - s * xb;
        A[row][b] = s * xa + c * xb;
        const double wa = W[row][a], wb = W[row][b];
        W[row][a] = c * wa - s * wb;
        W[row][b] = s * wa + c * wb;
      }
      __syncthreads();
      // rotate the round-robin order (perm[0] stays)
      if (tid == 0) {
        const int last = perm[P - 1];
        for (int i = P - 1; i > 1; --i) perm[i] = perm[i - 1];
        perm[1] = last;
      }
      __syncthreads();
    }
  }
  // sort descending (selection order, one thread: P <= 80)
  if (tid == 0) {
    int idx[P];
    for (int i = 0; i < P; ++i) idx[i] = i;
    for (int i = 0; i < P; ++i) {
      int best = i;
      for (int j = i + 1; j < P; ++j)
        if (A[idx[j]][idx[j]] > A[idx[best]][idx[best]]) best = j;
      const int t = idx[i]; idx[i] = idx[best]; idx[best] = t;
    }
    for (int i = 0; i < P; ++i) {
      lam_out[i] = fmax(A[idx[i]][idx[i]], 0.0);
      for (int row = 0; row < P; ++row) Wout[row * P + i] = W[row][idx[i]];
    }
  }
}

// A[i][rho] = lam^(1/4) (Q W)[i][rho]  and  B[rho][k] = lam^(-1/4) (Bt W)[k][rho],
// rounded to BF16 (zero where lam = 0); sigma[rho] = sqrt(lam).
template <int P>
__global__ void __launch_bounds__(kLrThreads) lr_factor_kernel(
    const float *__restrict__ Q, int M, const float *__restrict__ Bt, int K,
    const double *__restrict__ Wv, const double *__restrict__ lam, int r,
    uint16_t *__restrict__ U, uint16_t *__restrict__ V, float *__restrict__ sigma) {
  __shared__ float Ws[P][64];
  __shared__ float fa[64], fb[64];
  for (int e = threadIdx.x; e < P * r; e += kLrThreads) Ws[e / r][e % r] = (float)Wv[(e / r) * P + e % r];
  const double lmin = 1e-20 * lam[0];      // numerically zero below this
  for (int rho = threadIdx.x; rho < r; rho += kLrThreads) {
    const double l = lam[rho] > lmin ? lam[rho] : 0.0;
    fa[rho] = l > 0.0 ? (float)sqrt(sqrt(l)) : 0.f;
    fb[rho] = l > 0.0 ? (float)(1.0 / sqrt(sqrt(l))) : 0.f;
    if (blockIdx.x == 0 && sigma != nullptr) sigma[rho] = (float)sqrt(l);
  }
  __syncthreads();
  const long long total = (long long)M + K;
  for (long long row = (long long)blockIdx.x * kLrThreads + threadIdx.x; row < total;
       row += (long long)gridDim.x * kLrThreads) {
    const bool isU = row < M;
    const float *src = isU ? Q + row * P : Bt + (row - M) * P;
    float x[P];
#pragma unroll
    for (int j = 0; j < P; ++j) x[j] = src[j];
    for (int rho = 0; rho < r; ++rho) {
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < P; ++j) s = fmaf(x[j], Ws[j][rho], s);
      if (isU)
        U[row * r + rho] = f32_to_bf16_rn_bits(s * fa[rho]);
      else
        V[(size_t)rho * K + (row - M)] = f32_to_bf16_rn_bits(s * fb[rho]);
    }
  }
}

namespace {
int lr_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}
struct LrLayout {
  size_t X, Y, Z, mpart, part, chol, w, lam, total;
  int p, nparts;
};
int lr_p(int rank) { return rank + kLrOver <= 32 ? 32 : (rank + kLrOver <= 48 ? 48 : (rank + kLrOver <= 64 ? 64 : 80)); }

LrLayout lr_layout(int M, int K, int rank) {
  LrLayout L{};
  L.p = lr_p(rank);
  const int nmax = std::max(M, K);
  L.nparts = (nmax + kLrGramRows - 1) / kLrGramRows;
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += (b + 255) & ~(size_t)255;
    return o;
  };
  L.X = take((size_t)K * L.p * 4);          // X, then Z and Bt (K x p)
  L.Y = take((size_t)M * L.p * 4);          // Y / Q (M x p)
  L.Z = take((size_t)K * L.p * 4);          // Z (K x p)
  // split-product partials: at most one slice per kLrMinSlice of the inner
  // dimension for either product
  const size_t rows = std::max((size_t)((K + kLrMinSlice - 1) / kLrMinSlice) * M,
                               (size_t)((M + kLrMinSlice - 1) / kLrMinSlice) * K);
  L.mpart = take(rows * L.p * 4);
  L.part = take((size_t)L.nparts * L.p * L.p * 8);
  L.chol = take((size_t)L.p * L.p * 8);
  L.w = take((size_t)L.p * L.p * 8);
  L.lam = take((size_t)L.p * 8);
  L.total = off;
  return L;
}

template <int P>
cudaError_t lr_run(const LowrankArgs &a, const LrLayout &lay, cudaStream_t st, Launcher &L) {
  char *ws = static_cast<char *>(a.workspace);
  float *X = reinterpret_cast<float *>(ws + lay.X);
  float *Y = reinterpret_cast<float *>(ws + lay.Y);
  float *Z = reinterpret_cast<float *>(ws + lay.Z);
  double *part = reinterpret_cast<double *>(ws + lay.part);
  double *chol = reinterpret_cast<double *>(ws + lay.chol);
  double *W = reinterpret_cast<double *>(ws + lay.w);
  double *lam = reinterpret_cast<double *>(ws + lay.lam);
  float *mpart = reinterpret_cast<float *>(ws + lay.mpart);
  const int M = a.M, K = a.K;
  const size_t dyn = (size_t)2 * P * (P + 1) * sizeof(double);
  cudaError_t e;
  auto orth = [&](float *B, int n) -> cudaError_t {
    const int np = (n + kLrGramRows - 1) / kLrGramRows;
    for (int pass = 0; pass < 2; ++pass) {
      cudaError_t err;
      if ((err = L.launch("lr_gram", lr_gram_kernel<P>, dim3(np), dim3(kLrThreads), 0, st, false,
                          (const float *)B, n, part)) != cudaSuccess)
        return err;
      if ((err = L.launch("lr_chol", lr_chol_kernel<P>, dim3(1), dim3(kLrCholThreads), dyn, st,
                          false, (const double *)part, np, chol)) != cudaSuccess)
        return err;
      const int g = (n + kLrSolveThreads - 1) / kLrSolveThreads;
      if ((err = L.launch("lr_apply", lr_apply_solve_kernel<P>, dim3(g), dim3(kLrSolveThreads), 0,
                          st, false, B, n, (const double *)chol)) != cudaSuccess)
        return err;
    }
    return cudaSuccess;
  };
  // out = R in (TRANS 0, n = M) or R^T in (TRANS 1, n = K), split along the
  // inner dimension, then the slices summed in order
  auto mul = [&](auto kern, const float *in, float *out, int n, int inner) -> cudaError_t {
    // slice length: a multiple of kLrChunk in [kLrMinSlice, kLrSlice] (the
    // workspace holds the partials of the shortest), chosen so that the CTAs fill
    // whole waves of the resident slots as nearly as possible
    int occ = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kLrThreads, 0) != cudaSuccess ||
        occ < 1)
      occ = 1;
    const double slots = (double)lr_sm_count() * occ;
    const int tiles = (n + kLrTile - 1) / kLrTile;
    int best = kLrSlice;
    double best_eff = -1.0;
    for (int sl = kLrMinSlice; sl <= kLrSlice; sl += kLrChunk) {
      const int ns = (inner + sl - 1) / sl;
      const double waves = tiles * (double)ns / slots;
      const double eff = waves / std::ceil(waves);
      if (eff > best_eff + 1e-9) { best_eff = eff; best = sl; }
    }
    const int ns = (inner + best - 1) / best;
    cudaError_t err = L.launch("lr_mul", kern, dim3(tiles, ns), dim3(kLrThreads), 0, st, false,
                               a.R, in, mpart, M, K, best);
    if (err != cudaSuccess) return err;
    const long long cnt = (long long)n * P;
    return L.launch("lr_reduce", lr_reduce_kernel, dim3(148 * 4), dim3(256), 0, st, false,
                    (const float *)mpart, ns, cnt, out);
  };
  auto rx = [&](const float *in, float *out) { return mul(lr_mul_kernel<P, 0>, in, out, M, K); };
  auto rtq = [&](const float *in, float *out) { return mul(lr_mul_kernel<P, 1>, in, out, K, M); };
  if ((e = L.launch("lr_gaussian", lr_gaussian_kernel, dim3(148 * 4), dim3(256), 0, st, false, X,
                    (long long)K * P, (uint64_t)a.seed)) != cudaSuccess)
    return e;
  if ((e = rx(X, Y)) != cudaSuccess || (e = orth(Y, M)) != cudaSuccess) return e;
  for (int it = 0; it < a.iters; ++it) {
    if ((e = rtq(Y, Z)) != cudaSuccess || (e = orth(Z, K)) != cudaSuccess) return e;
    if ((e = rx(Z, Y)) != cudaSuccess || (e = orth(Y, M)) != cudaSuccess) return e;
  }
  if ((e = rtq(Y, Z)) != cudaSuccess) return e;          // Bt = R^T Q
  const int np = (K + kLrGramRows - 1) / kLrGramRows;
  if ((e = L.launch("lr_gram", lr_gram_kernel<P>, dim3(np), dim3(kLrThreads), 0, st, false,
                    (const float *)Z, K, part)) != cudaSuccess)
    return e;
  if ((e = L.launch("lr_eig", lr_eig_kernel<P>, dim3(1), dim3(kLrThreads), dyn, st, false,
                    (const double *)part, np, W, lam)) != cudaSuccess)
    return e;
  const int g = std::max(1, std::min((M + K + kLrThreads - 1) / kLrThreads, 148 * 4));
  return L.launch("lr_factor", lr_factor_kernel<P>, dim3(g), dim3(kLrThreads), 0, st, false,
                  (const float *)Y, M, (const float *)Z, K, (const double *)W,
                  (const double *)lam, a.rank, a.U, a.V, a.sigma);
}
}  // namespace

size_t lowrank_workspace_bytes(int M, int K, int rank) { return lr_layout(M, K, rank).total; }

cudaError_t prepare_lowrank_kernels() {
  cudaError_t e;
#define LR_ATTR(P)                                                                            \
  for (const void *f : {(const void *)lr_chol_kernel<P>, (const void *)lr_eig_kernel<P>})      \
    if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                  2 * P * (P + 1) * (int)sizeof(double))) != cudaSuccess)     \
      return e;
  LR_ATTR(32) LR_ATTR(48) LR_ATTR(64) LR_ATTR(80)
#undef LR_ATTR
  return cudaSuccess;
}

cudaError_t launch_lowrank(const LowrankArgs &a, cudaStream_t st, Launcher &L) {
  const LrLayout lay = lr_layout(a.M, a.K, a.rank);
  switch (lay.p) {
    case 32: return lr_run<32>(a, lay, st, L);
    case 48: return lr_run<48>(a, lay, st, L);
    case 64: return lr_run<64>(a, lay, st, L);
    default: return lr_run<80>(a, lay, st, L);
  }
}

}  // namespace dvssq
