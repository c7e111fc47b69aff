// Blockwise Walsh-Hadamard transform by a group of P = b/16 threads.
//
// Sylvester's H_b factors as H_16 (x) H_P over the split n = P*a + t of the
// element index (a in [0,16), t in [0,P)): thread t first loads x[P*a + t]
// for all a and applies H_16 along a in registers, the group transposes the
// 16 x P intermediate through padded shared memory, and each thread then
// applies H_P along t.  Thread t ends up holding the outputs 16t .. 16t+15
// (contiguous), unscaled (the 1/sqrt(b) factor is applied by the caller).
#pragma once

namespace dvssq {

template <typename T>
__device__ __forceinline__ void hadamard_inplace(T *v, int n) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
    if (h >= n) break;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < n && !(i & h)) {
        T a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

template <typename T>
__device__ __forceinline__ void h16(T v[16]) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (!(i & h)) {
        T a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

template <typename T>
__device__ __forceinline__ void h8(T *v) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (!(i & h)) {
        T a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

// Scratch elements per group: a 16 x (P+1) padded matrix plus one element
// that staggers consecutive groups across banks.
template <int B>
struct GroupScratch {
  static constexpr int P = B / 16;
  static constexpr int kElems = 16 * (P + 1) + 1;
};

// v[a] = x[P*a + t] on entry; v[j] = (S_b x)[16t + j] on exit.  All P threads
// of the group (which lives inside one warp) must call it together; the
// whole warp calls __syncwarp.
template <int B, typename T>
__device__ __forceinline__ void fwht_group(T v[16], T *scratch, int t) {
  constexpr int P = B / 16;
  static_assert(B == 128 || B == 256, "Hadamard block must be 128 or 256");
  h16(v);
#pragma unroll
  for (int a = 0; a < 16; ++a) scratch[a * (P + 1) + t] = v[a];
  __syncwarp();
  if constexpr (P == 16) {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = scratch[t * (P + 1) + j];
    h16(v);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[j] = scratch[(2 * t) * (P + 1) + j];
      v[8 + j] = scratch[(2 * t + 1) * (P + 1) + j];
    }
    h8(v);
    h8(v + 8);
  }
  __syncwarp();
}

}  // namespace dvssq
