// Allocation-free decode forward: the workspace of dvssq_linear_forward's
// decode path lives in a fixed device array of this library instead of a
// caller-provided buffer (see dvssq_linear_forward_static in dvssq.h).
#include <cuda_runtime.h>

#include <mutex>
#include <string>
#include <vector>

#include "../../include/dvssq.h"
#include "kernels.h"

namespace dvssq {

// One per GPU that loads the library, held until the process exits.  In host
// code this name is only a host-side stand-in: kernels get the device address
// that static_scratch_ptr() looks up.
static __device__ __align__(256) unsigned char g_static_scratch[DVSSQ_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch on the current device, looked up once
// per device with that device current and kept for the life of the process
// (the library's other per-device set-up is kept the same way, so neither
// survives a cudaDeviceReset).
static cudaError_t static_scratch_ptr(void **out) {
  static std::mutex mu;
  static std::vector<void *> ptrs;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if ((int)ptrs.size() <= dev) ptrs.resize(dev + 1, nullptr);
  if (ptrs[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return cudaSuccess;
}

}  // namespace dvssq

extern "C" dvssq_status dvssq_linear_forward_static(const dvssq_shape *shape,
                                                    const dvssq_weights *w, const void *x,
                                                    int64_t T, const void *bias, void *y,
                                                    int32_t y_dtype, void *stream) {
  using namespace dvssq;
  if (T > 16) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  size_t need = 0;
  dvssq_status s = dvssq_forward_workspace_size(shape, T < 0 ? 0 : T, DVSSQ_PATH_DECODE, &need);
  if (s != DVSSQ_OK) return s;
  if (T == 0) return DVSSQ_OK;
  if (need > (size_t)DVSSQ_STATIC_SCRATCH_BYTES) {
    set_last_error("decode scratch of " + std::to_string(need) + " bytes exceeds the static " +
                   "scratch of " + std::to_string((size_t)DVSSQ_STATIC_SCRATCH_BYTES) + " bytes");
    return DVSSQ_ERR_WORKSPACE;
  }
  // the device check comes first: an unsupported device reports
  // DVSSQ_ERR_DEVICE, not a failed symbol lookup
  if ((s = ensure_device()) != DVSSQ_OK) return s;
  void *scratch = nullptr;
  cudaError_t e = static_scratch_ptr(&scratch);
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return DVSSQ_ERR_CUDA;
  }
  // dvssq_linear_forward validates the remaining arguments on the host
  // before any launch
  return dvssq_linear_forward(shape, w, x, T, bias, y, y_dtype, DVSSQ_PATH_DECODE, scratch,
                              (size_t)DVSSQ_STATIC_SCRATCH_BYTES, stream);
}
