// Activation rotation x_rot = H_K x (MiniCPM5-2B-Hadamard-GSQ card,
// Mathematical Foundations §1: X' = X H; Spark-X2.5-4B-Hadamard-GSQ card,
// Tier B: H_K = diag(H_b, ..., H_b)).
//
// One warp per b-element row-block: each lane loads b/32 contiguous BF16
// values with one vector load, applies the butterflies of the low index bits
// in registers and the five lane-index bits with shuffles, and stores fp32.
// HBM-bound: 2 B read + 4 B written per element.
#include "common.cuh"
#include "kernels.h"

namespace dvssq {

template <int B>
__global__ void __launch_bounds__(256) fwht_rows_kernel(const uint16_t *__restrict__ x,
                                                        float *__restrict__ y, long long nblk,
                                                        int cols, float c) {
  constexpr int EPL = B / 32;                 // elements per lane: 8 or 4
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long wb = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); wb < nblk;
       wb += warps) {
    const size_t off = (size_t)wb * B + (size_t)lane * EPL;   // row-blocks are contiguous
    float v[EPL];
    if constexpr (EPL == 8) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(x + off));
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
      }
    } else {
      const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(x + off));
      const uint32_t w[2] = {raw.x, raw.y};
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
      }
    }
#pragma unroll
    for (int h = 1; h < EPL; h <<= 1)
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (!(i & h)) {
          const float a = v[i], b = v[i + h];
          v[i] = a + b;
          v[i + h] = a - b;
        }
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const bool upper = lane & d;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const float p = __shfl_xor_sync(0xffffffffu, v[i], d);
        v[i] = upper ? (p - v[i]) : (v[i] + p);
      }
    }
    float4 *dst = reinterpret_cast<float4 *>(y + off);
#pragma unroll
    for (int i = 0; i < EPL; i += 4)
      dst[i / 4] = make_float4(v[i] * c, v[i + 1] * c, v[i + 2] * c, v[i + 3] * c);
  }
}

cudaError_t launch_fwht(const uint16_t *x, float *y, int64_t rows, int cols, int block,
                        cudaStream_t st, Launcher &L) {
  const long long nblk = (long long)rows * (cols / block);
  const float c = (float)sqrt(1.0 / (double)block);
  long long ctas = (nblk + 7) / 8;
  if (ctas > 148LL * 16) ctas = 148LL * 16;
  if (block == 256)
    return L.launch("fwht", fwht_rows_kernel<256>, dim3((unsigned)ctas), dim3(256), 0, st, false,
                    x, y, nblk, cols, c);
  return L.launch("fwht", fwht_rows_kernel<128>, dim3((unsigned)ctas), dim3(256), 0, st, false, x,
                  y, nblk, cols, c);
}

}  // namespace dvssq
