// Gated GELU between the up and down projections of a Spark-shaped MLP
// block ("Myric/Spark-X2.5-4B-GGUF", "The model": GELU FFN; "Spark-X2.5-4B-
// ASHQ1-GGUF", "Architecture": ffn_gate / ffn_up / ffn_down):
//     h = RN_bf16( gelu(g) * u ),  gelu(v) = v/2 (1 + erf(v / sqrt 2)),
// with g, u and h BF16 (hidden states are BF16 between layers) and the
// product formed in FP32.  Elementwise and HBM-bound: 6 bytes per element;
// eight elements per thread with 16-byte loads and stores.
#include "common.cuh"
#include "kernels.h"

namespace dvssq {

__global__ void __launch_bounds__(256) gelu_mul_kernel(const uint16_t *__restrict__ g,
                                                       const uint16_t *__restrict__ u,
                                                       uint16_t *__restrict__ h, long long n) {
  const long long n8 = n / 8;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 gv = __ldg(reinterpret_cast<const uint4 *>(g) + i);
    const uint4 uv = __ldg(reinterpret_cast<const uint4 *>(u) + i);
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a = gelu_erf(bf16_bits_to_f32(gw[q] & 0xFFFFu)) * bf16_bits_to_f32(uw[q] & 0xFFFFu);
      const float b = gelu_erf(bf16_bits_to_f32(gw[q] >> 16)) * bf16_bits_to_f32(uw[q] >> 16);
      o[q] = (uint32_t)f32_to_bf16_rn_bits(a) | ((uint32_t)f32_to_bf16_rn_bits(b) << 16);
    }
    reinterpret_cast<uint4 *>(h)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  // the last n % 8 elements
  for (long long i = n8 * 8 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    h[i] = f32_to_bf16_rn_bits(gelu_erf(bf16_bits_to_f32(g[i])) * bf16_bits_to_f32(u[i]));
}

cudaError_t launch_gelu_mul(const uint16_t *g, const uint16_t *u, uint16_t *h, long long n,
                            cudaStream_t st, Launcher &L) {
  const long long work = (n + 7) / 8;
  const int grid = (int)std::max(1LL, std::min((work + 255) / 256, 148LL * 8));
  return L.launch("gelu_mul", gelu_mul_kernel, dim3(grid), dim3(256), 0, st, false, g, u, h, n);
}

}  // namespace dvssq
