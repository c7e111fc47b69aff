// KV-BSS attention for decode (Spark-X2.5-4B-Hadamard-GSQ model card, "2.
// KV-BSS: Key-Value Binding Softmax Sharpening": focus factor scaling of the
// logits by tau_focus = 1.10 and attention haze truncation, every logit more
// than 12 nats below the maximum masked to -inf before the softmax):
//
//   s_l = (q . k_l) tau / sqrt(d),  m = max_l s_l,
//   p_l = exp(s_l - m) if s_l >= m - haze else 0,   out = sum_l p_l v_l / sum_l p_l
//
// for one query token per sequence and query head, over a BF16 KV cache
// with grouped-query heads (G = Hq / Hkv query heads share a KV head).  The
// threshold depends on the final maximum, so the work is split in two
// passes over the context, both HBM-bound:
//   bss_logits  per (256-key chunk, KV head, sequence): the G query heads'
//               logits of the chunk (FP32 dot products: each lane holds d/32
//               dimensions, eight keys' partial sums are reduce-scattered so
//               that every lane ends with one (key, head) logit), stored with
//               the chunk's maximum per head;
//   bss_pv      the global maximum from the chunk maxima, the masked weights
//               of the chunk, and the chunk's partial sum p v; the V row of a
//               key that the haze mask drops for all G heads is never read;
//   bss_merge   out = sum over chunks of the partials / sum of the weights,
//               in chunk order (deterministic).
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace dvssq {

constexpr int kBssChunk = 256;        // keys per CTA
constexpr int kBssThreads = 256;
constexpr int kBssWarps = kBssThreads / 32;
static_assert(kBssChunk == kBssThreads, "one key of the chunk per thread when forming the weights");

struct BssParams {
  const uint16_t *q, *k, *v;          // BF16: q [B][Hq][d], k/v [B][Hkv][L][d]
  float *out;                         // FP32 [B][Hq][d]
  float *logit;                       // [B][Hq][L]
  float *cmax;                        // [B][Hq][nc]
  float *psum;                        // [B][Hq][nc]
  float *pacc;                        // [B][Hq][nc][d]
  int B, Hq, Hkv, L, nc;
  float scale, haze;                  // tau / sqrt(d); haze <= 0: no truncation
};

// 8 BF16 values (16 bytes) or 4 (8 bytes) to FP32
template <int DL>
__device__ __forceinline__ void bss_load_row(const uint16_t *src, float *f) {
  if constexpr (DL == 8) {
    const uint4 u = *reinterpret_cast<const uint4 *>(src);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const uint2 u = *reinterpret_cast<const uint2 *>(src);
    const uint32_t w[2] = {u.x, u.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// Logits of one chunk: warp w takes batches of KPW = 32 / G consecutive keys
// (batch j of the chunk at keys 8 j KPW + w KPW ...).
template <int D, int G>
__global__ void __launch_bounds__(kBssThreads) bss_logits_kernel(const BssParams p) {
  constexpr int DL = D / 32;               // dimensions per lane
  constexpr int KPW = 32 / G;              // keys per batch: KPW * G = 32 values per lane
  constexpr int NB = kBssChunk / (KPW * kBssWarps);   // batches per warp
  __shared__ float lg[G][kBssChunk];
  __shared__ float wmax[kBssWarps][G];
  const int c = blockIdx.x, kh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = p.L, key0 = c * kBssChunk;
  // this lane's dimensions of the G query heads, pre-scaled
  float qv[G][DL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float f[DL];
    bss_load_row<DL>(p.q + ((size_t)b * p.Hq + kh * G + g) * D + lane * DL, f);
#pragma unroll
    for (int i = 0; i < DL; ++i) qv[g][i] = f[i] * p.scale;
  }
  const uint16_t *kbase = p.k + ((size_t)b * p.Hkv + kh) * (size_t)L * D + lane * DL;
  float mymax = -INFINITY;   // max of this lane's logits (head lane % G)
#pragma unroll 1
  for (int nb = 0; nb < NB; ++nb) {
    const int kb0 = key0 + (nb * kBssWarps + warp) * KPW;
    float part[32];
    float kf[KPW][DL];
#pragma unroll
    for (int j = 0; j < KPW; ++j) {
      if (kb0 + j < L) bss_load_row<DL>(kbase + (size_t)(kb0 + j) * D, kf[j]);
      else {
#pragma unroll
        for (int i = 0; i < DL; ++i) kf[j][i] = 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < KPW; ++j)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < DL; ++i) s = fmaf(qv[g][i], kf[j][i], s);
        part[j * G + g] = s;
      }
    // reduce-scatter over the 32 lanes: after the stage with offset o the
    // lane keeps the half whose index bit log2(o) equals its lane bit
#pragma unroll
    for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
      const bool hi = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const float send = hi ? part[i] : part[i + n / 2];
        const float keep = hi ? part[i + n / 2] : part[i];
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    // lane holds the logit of value index `lane` = key lane / G, head lane % G
    const int j = lane / G, g = lane % G;
    const bool valid = kb0 + j < L;
    lg[g][kb0 + j - key0] = valid ? part[0] : -INFINITY;
    if (valid) mymax = fmaxf(mymax, part[0]);
  }
  // per-head maximum: lanes with the same lane % G hold the same head
#pragma unroll
  for (int o = G; o < 32; o <<= 1) mymax = fmaxf(mymax, __shfl_xor_sync(0xffffffffu, mymax, o));
  if (lane < G) wmax[warp][lane] = mymax;
  __syncthreads();
  // logits out, coalesced
  for (int i = tid; i < G * kBssChunk; i += kBssThreads) {
    const int g = i / kBssChunk, kk = i - g * kBssChunk;
    if (key0 + kk < L) p.logit[((size_t)b * p.Hq + kh * G + g) * L + key0 + kk] = lg[g][kk];
  }
  if (tid < G) {
    float m = -INFINITY;
    for (int w = 0; w < kBssWarps; ++w) m = fmaxf(m, wmax[w][tid]);
    p.cmax[((size_t)b * p.Hq + kh * G + tid) * p.nc + c] = m;
  }
}

// Masked weights and the partial p . V of one chunk.
template <int D, int G>
__global__ void __launch_bounds__(kBssThreads, 3) bss_pv_kernel(const BssParams p) {
  constexpr int DL = D / 32;
  __shared__ float pw[G][kBssChunk];
  __shared__ float s_m[G];
  __shared__ float red[kBssWarps][G][D];      // per-warp partial p v
  __shared__ float lsum[kBssWarps][G];
  const int c = blockIdx.x, kh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = p.L, key0 = c * kBssChunk;
  pdl_wait();                                  // logits and chunk maxima of bss_logits
  // global maximum per head from the chunk maxima
  if (warp < G) {
    const float *cm = p.cmax + ((size_t)b * p.Hq + kh * G + warp) * p.nc;
    float m = -INFINITY;
#pragma unroll 8
    for (int i = lane; i < p.nc; i += 32) m = fmaxf(m, cm[i]);
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_m[warp] = m;
  }
  __syncthreads();
  {
    // G logits per thread, loaded together
    float sv[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
      sv[g] = key0 + tid < L ? p.logit[((size_t)b * p.Hq + kh * G + g) * L + key0 + tid] : 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float m = s_m[g];
      pw[g][tid] = key0 + tid < L && (p.haze <= 0.f || sv[g] >= m - p.haze) ? expf(sv[g] - m) : 0.f;
    }
  }
  __syncthreads();
  float acc[G][DL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int i = 0; i < DL; ++i) acc[g][i] = 0.f;
  float lw[G];
#pragma unroll
  for (int g = 0; g < G; ++g) lw[g] = 0.f;
  const uint16_t *vbase = p.v + ((size_t)b * p.Hkv + kh) * (size_t)L * D + lane * DL;
  // warp w: keys w + 8 j of the chunk in groups of KG, software-pipelined:
  // the raw V rows of the next group are in flight while the current group
  // is weighted and added.  A key dropped for every head is skipped without
  // reading its V row.
  using Raw = typename std::conditional<DL == 8, uint4, uint2>::type;
  constexpr int KG = 2;                                    // keys per group
  constexpr int NGRP = kBssChunk / (kBssWarps * KG);       // groups per warp
  Raw raw[2][KG];
  auto issue = [&](int grp, Raw *dst) {
#pragma unroll
    for (int u = 0; u < KG; ++u) {
      const int kk = warp + kBssWarps * (KG * grp + u);
      bool any = false;
#pragma unroll
      for (int g = 0; g < G; ++g) any |= pw[g][kk] != 0.f;
      if (any) dst[u] = *reinterpret_cast<const Raw *>(vbase + (size_t)(key0 + kk) * D);
    }
  };
  auto consume = [&](int grp, const Raw *src) {
#pragma unroll
    for (int u = 0; u < KG; ++u) {
      const int kk = warp + kBssWarps * (KG * grp + u);
      float wt[G];
      bool any = false;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        wt[g] = pw[g][kk];
        any |= wt[g] != 0.f;
      }
      if (!any) continue;
      float vf[DL];
      if constexpr (DL == 8) {
        const uint32_t w[4] = {src[u].x, src[u].y, src[u].z, src[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          vf[2 * i] = __uint_as_float(w[i] << 16);
          vf[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
      } else {
        const uint32_t w[2] = {src[u].x, src[u].y};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          vf[2 * i] = __uint_as_float(w[i] << 16);
          vf[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        lw[g] += wt[g];
#pragma unroll
        for (int i = 0; i < DL; ++i) acc[g][i] = fmaf(wt[g], vf[i], acc[g][i]);
      }
    }
  };
  static_assert(NGRP % 2 == 0, "groups go in pairs (double buffer)");
  issue(0, raw[0]);
#pragma unroll 1
  for (int grp = 0; grp < NGRP; grp += 2) {
    issue(grp + 1, raw[1]);
    consume(grp, raw[0]);
    if (grp + 2 < NGRP) issue(grp + 2, raw[0]);
    consume(grp + 1, raw[1]);
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int i = 0; i < DL; ++i) red[warp][g][lane * DL + i] = acc[g][i];
    if (lane == 0) lsum[warp][g] = lw[g];
  }
  __syncthreads();
  // warps' partials added in warp order
  for (int i = tid; i < G * D; i += kBssThreads) {
    const int g = i / D, dd = i - g * D;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kBssWarps; ++w) s += red[w][g][dd];
    p.pacc[(((size_t)b * p.Hq + kh * G + g) * p.nc + c) * D + dd] = s;
  }
  if (tid < G) {
    float s = 0.f;
    for (int w = 0; w < kBssWarps; ++w) s += lsum[w][tid];
    p.psum[((size_t)b * p.Hq + kh * G + tid) * p.nc + c] = s;
  }
}

// out[b][h][:] = sum_c pacc / sum_c psum, chunks in order: thread (j, dd)
// sums the j-th quarter of the chunks for dimension dd (loads in batches
// of 16 in flight), and the quarters are added in order.
template <int D>
__global__ void __launch_bounds__(4 * D) bss_merge_kernel(const BssParams p) {
  __shared__ float ps[4][D], ls[4];
  const int h = blockIdx.x, b = blockIdx.y, dd = threadIdx.x % D, j = threadIdx.x / D;
  pdl_wait();
  const size_t row = (size_t)b * p.Hq + h;
  const int c0 = (j * p.nc) / 4, c1 = ((j + 1) * p.nc) / 4;
  float l = 0.f, s = 0.f;
  for (int cb = c0; cb < c1; cb += 16) {
    float lv[16], sv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const bool in = cb + u < c1;
      lv[u] = in && dd == 0 ? p.psum[row * p.nc + cb + u] : 0.f;
      sv[u] = in ? p.pacc[(row * p.nc + cb + u) * D + dd] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      l += lv[u];
      s += sv[u];
    }
  }
  ps[j][dd] = s;
  if (dd == 0) ls[j] = l;
  __syncthreads();
  if (j == 0) {
    const float lt = ((ls[0] + ls[1]) + ls[2]) + ls[3];
    p.out[row * D + dd] = (((ps[0][dd] + ps[1][dd]) + ps[2][dd]) + ps[3][dd]) / lt;
  }
}

namespace {
struct BssLayout {
  size_t logit, cmax, psum, pacc, total;
};
BssLayout bss_layout(int B, int Hq, int L, int D) {
  const size_t nc = (size_t)(L + kBssChunk - 1) / kBssChunk;
  BssLayout y{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  y.logit = take((size_t)B * Hq * L * 4);
  y.cmax = take((size_t)B * Hq * nc * 4);
  y.psum = take((size_t)B * Hq * nc * 4);
  y.pacc = take((size_t)B * Hq * nc * D * 4);
  y.total = off;
  return y;
}

template <int D, int G>
cudaError_t bss_run(const BssParams &p, cudaStream_t st, Launcher &L) {
  const dim3 grid((unsigned)p.nc, (unsigned)p.Hkv, (unsigned)p.B);
  cudaError_t e = L.launch("bss_logits", bss_logits_kernel<D, G>, grid, dim3(kBssThreads), 0, st,
                           false, p);
  if (e != cudaSuccess) return e;
  e = L.launch("bss_pv", bss_pv_kernel<D, G>, grid, dim3(kBssThreads), 0, st, true, p);
  if (e != cudaSuccess) return e;
  return L.launch("bss_merge", bss_merge_kernel<D>, dim3((unsigned)p.Hq, (unsigned)p.B),
                  dim3(4 * D), 0, st, true, p);
}
}  // namespace

size_t bss_workspace_bytes(int B, int Hq, int L, int D) { return bss_layout(B, Hq, L, D).total; }

cudaError_t launch_bss_attention(const BssArgs &a, cudaStream_t st, Launcher &L) {
  const BssLayout y = bss_layout(a.B, a.Hq, a.L, a.D);
  char *ws = static_cast<char *>(a.workspace);
  BssParams p{};
  p.q = a.q; p.k = a.k; p.v = a.v; p.out = a.out;
  p.logit = reinterpret_cast<float *>(ws + y.logit);
  p.cmax = reinterpret_cast<float *>(ws + y.cmax);
  p.psum = reinterpret_cast<float *>(ws + y.psum);
  p.pacc = reinterpret_cast<float *>(ws + y.pacc);
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.L = a.L;
  p.nc = (a.L + kBssChunk - 1) / kBssChunk;
  p.scale = a.tau / sqrtf((float)a.D);
  p.haze = a.haze;
  const int G = a.Hq / a.Hkv;
#define BSS_CASE(D_, G_) \
  if (a.D == D_ && G == G_) return bss_run<D_, G_>(p, st, L);
  BSS_CASE(256, 2) BSS_CASE(256, 4)
  BSS_CASE(128, 2) BSS_CASE(128, 4) BSS_CASE(128, 8)
#undef BSS_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dvssq
