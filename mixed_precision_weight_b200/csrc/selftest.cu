// Bounded-wait self-test: a kernel that waits on something nothing will
// ever signal, through the same helpers the GEMV, GEMM and stack kernels
// use, so that a test can watch a wait run out and the call return with the
// device error word set (no fault, no trap: the wait simply gives up).
#include "common.cuh"
#include "kernels.h"

namespace dvssq {

// A counter nobody increments (the grid-barrier form of the wait).
__device__ unsigned int g_selftest_counter = 0;

__global__ void __launch_bounds__(32) selftest_wait_kernel(int which) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t err0 = *(volatile uint32_t *)&g_dvssq_error;
  if (which == 0) {
    // an mbarrier expecting one arrival that never comes
    mbar_init(&bar, 1);
    fence_mbarrier_init();
    mbar_wait(&bar, 0);
  } else {
    counter_wait(&g_selftest_counter, 1u, err0);
  }
}

cudaError_t set_wait_limit(long long cycles) {
  const long long v = cycles > 0 ? cycles : kWaitLimitCycles;
  return cudaMemcpyToSymbol(g_wait_limit, &v, sizeof(v));
}

cudaError_t launch_selftest_wait(int which, cudaStream_t st, Launcher &L) {
  return L.launch("selftest_wait", selftest_wait_kernel, dim3(1), dim3(32), 0, st, false, which);
}

}  // namespace dvssq

extern "C" dvssq_status dvssq_set_wait_limit(int64_t cycles) {
  using namespace dvssq;
  dvssq_status s = ensure_device();
  if (s != DVSSQ_OK) return s;
  const cudaError_t e = set_wait_limit((long long)cycles);
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

extern "C" dvssq_status dvssq_selftest_wait(int32_t which, void *stream) {
  using namespace dvssq;
  if (which != 0 && which != 1) return DVSSQ_ERR_INVALID_ARG;
  dvssq_status s = ensure_device();
  if (s != DVSSQ_OK) return s;
  const cudaError_t e =
      launch_selftest_wait(which, static_cast<cudaStream_t>(stream), launcher());
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}
