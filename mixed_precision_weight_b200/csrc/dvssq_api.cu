// C ABI of libdvssq.so (declared in include/dvssq.h): host-side validation,
// workspace sizing, device checks, per-kernel profiling and dispatch to the
// kernel launchers.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "../../include/dvssq.h"
#include "common.cuh"
#include "kernels.h"

namespace dvssq {


Launcher &launcher() {
  static Launcher L;
  return L;
}

namespace {

thread_local std::string t_last_error;

struct ProfileTotal {
  const char *name;
  int64_t launches;
  double ms;
};
std::mutex g_prof_mu;
std::vector<ProfileTotal> g_prof;

dvssq_status cuda_fail(cudaError_t e) {
  t_last_error = cudaGetErrorString(e);
  return DVSSQ_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// Shape rules shared by every entry point (see dvssq_shape in dvssq.h).
dvssq_status check_shape(const dvssq_shape *s) {
  if (s == nullptr) return DVSSQ_ERR_INVALID_ARG;
  if (s->M < 1 || s->K < 1 || s->n_sal < 0 || s->rank < 0) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (s->M > (1 << 24) || s->K > 65536) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (s->block != 128 && s->block != 256) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (s->group != 64) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (s->K % s->block != 0) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (s->n_sal > s->K || s->n_sal % 16 != 0 || s->n_sal > kMaxSalient)
    return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  // U rows travel as 16-byte vectors of 8 BF16 values
  if (s->rank > 64 || s->rank % 8 != 0) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  return DVSSQ_OK;
}

// Per-device one-time set-up: capability check and kernel attributes.
dvssq_status ensure_device() {
  static std::mutex mu;
  static std::vector<int> ready;   // 0 unknown, 1 ok, -1 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lk(mu);
  if ((int)ready.size() <= dev) ready.resize(dev + 1, 0);
  if (ready[dev] == 1) return DVSSQ_OK;
  if (ready[dev] == -1) return DVSSQ_ERR_DEVICE;
  int major = 0, minor = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
    return cuda_fail(e);
  if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
    return cuda_fail(e);
  if (major != 10 || minor != 0) {
    ready[dev] = -1;
    t_last_error = "libdvssq is built for sm_100a (compute capability 10.0) only";
    return DVSSQ_ERR_DEVICE;
  }
  if ((e = prepare_encode_kernels()) != cudaSuccess) return cuda_fail(e);
  if ((e = prepare_forward_kernels()) != cudaSuccess) return cuda_fail(e);
  if ((e = prepare_stack_kernels()) != cudaSuccess) return cuda_fail(e);
  if ((e = prepare_materialize_kernels()) != cudaSuccess) return cuda_fail(e);
  if ((e = prepare_lowrank_kernels()) != cudaSuccess) return cuda_fail(e);
  ready[dev] = 1;
  return DVSSQ_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tiled_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

void set_last_error(const std::string &msg) { t_last_error = msg; }

CUresult encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                        uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                        uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = tiled_encoder();
  if (fn == nullptr) return CUDA_ERROR_NOT_FOUND;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

cudaError_t prepare_decode_kernels();
cudaError_t prepare_prefill_kernels();

cudaError_t prepare_forward_kernels() {
  cudaError_t e = prepare_decode_kernels();
  if (e != cudaSuccess) return e;
  return prepare_prefill_kernels();
}

static int choose_path(int32_t path, int64_t T) {
  if (path == DVSSQ_PATH_DECODE) return DVSSQ_PATH_DECODE;
  if (path == DVSSQ_PATH_PREFILL) return DVSSQ_PATH_PREFILL;
  return T <= 16 ? DVSSQ_PATH_DECODE : DVSSQ_PATH_PREFILL;
}

}  // namespace dvssq

using namespace dvssq;

extern "C" {

int32_t dvssq_abi_version(void) { return DVSSQ_ABI_VERSION; }

const char *dvssq_status_string(dvssq_status s) {
  switch (s) {
    case DVSSQ_OK: return "ok";
    case DVSSQ_ERR_INVALID_ARG: return "invalid argument";
    case DVSSQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DVSSQ_ERR_MISALIGNED: return "buffer not 16-byte aligned (workspace: 256-byte)";
    case DVSSQ_ERR_WORKSPACE: return "workspace too small";
    case DVSSQ_ERR_CUDA: return "CUDA error";
    case DVSSQ_ERR_DEVICE: return "unsupported device (needs compute capability 10.0)";
  }
  return "unknown status";
}

const char *dvssq_last_error(void) { return t_last_error.c_str(); }

dvssq_status dvssq_fwht(const void *x, float *y, int64_t rows, int32_t cols, int32_t block,
                        void *stream) {
  if (rows < 0 || cols < 1 || cols > (1 << 24)) return DVSSQ_ERR_INVALID_ARG;
  if (block != 128 && block != 256) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (cols % block != 0) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return DVSSQ_OK;
  if (x == nullptr || y == nullptr) return DVSSQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return DVSSQ_ERR_MISALIGNED;
  dvssq_status s = ensure_device();
  if (s != DVSSQ_OK) return s;
  cudaError_t e = launch_fwht(static_cast<const uint16_t *>(x), y, rows, cols, block,
                              static_cast<cudaStream_t>(stream), launcher());
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

dvssq_status dvssq_gelu_mul(const void *gate, const void *up, void *h, int64_t n, void *stream) {
  if (n < 0 || n > ((int64_t)1 << 40)) return DVSSQ_ERR_INVALID_ARG;
  if (n == 0) return DVSSQ_OK;
  if (gate == nullptr || up == nullptr || h == nullptr) return DVSSQ_ERR_INVALID_ARG;
  if (!aligned16(gate) || !aligned16(up) || !aligned16(h)) return DVSSQ_ERR_MISALIGNED;
  dvssq_status s = ensure_device();
  if (s != DVSSQ_OK) return s;
  cudaError_t e = launch_gelu_mul(static_cast<const uint16_t *>(gate),
                                  static_cast<const uint16_t *>(up), static_cast<uint16_t *>(h),
                                  n, static_cast<cudaStream_t>(stream), launcher());
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

dvssq_status dvssq_encode_workspace_size(const dvssq_shape *shape, size_t *bytes) {
  dvssq_status s = check_shape(shape);
  if (s != DVSSQ_OK) return s;
  if (bytes == nullptr) return DVSSQ_ERR_INVALID_ARG;
  *bytes = encode_workspace_bytes(shape->M, shape->K, shape->block, shape->n_sal);
  return DVSSQ_OK;
}

dvssq_status dvssq_encode(const dvssq_shape *shape, const void *W, const float *act_scale,
                          const dvssq_weights *out, float *resid, dvssq_encode_info *info,
                          void *workspace, size_t workspace_bytes, void *stream) {
  dvssq_status s = check_shape(shape);
  if (s != DVSSQ_OK) return s;
  if (W == nullptr || act_scale == nullptr || out == nullptr || workspace == nullptr)
    return DVSSQ_ERR_INVALID_ARG;
  if (out->q4 == nullptr || out->s4 == nullptr || out->s8 == nullptr) return DVSSQ_ERR_INVALID_ARG;
  if (shape->n_sal > 0 && (out->sal_idx == nullptr || out->q8 == nullptr))
    return DVSSQ_ERR_INVALID_ARG;
  const void *bufs[] = {W, act_scale, out->q4, out->s4, out->s8, resid, out->sal_idx, out->q8};
  for (const void *b : bufs)
    if (b != nullptr && !aligned16(b)) return DVSSQ_ERR_MISALIGNED;
  if (!aligned256(workspace)) return DVSSQ_ERR_MISALIGNED;
  if (workspace_bytes < encode_workspace_bytes(shape->M, shape->K, shape->block, shape->n_sal))
    return DVSSQ_ERR_WORKSPACE;
  if ((s = ensure_device()) != DVSSQ_OK) return s;
  EncodeArgs a;
  a.M = shape->M; a.K = shape->K; a.block = shape->block; a.n_sal = shape->n_sal;
  a.W = W; a.act_scale = act_scale;
  a.q4 = out->q4; a.s4 = out->s4; a.sal_idx = out->sal_idx; a.q8 = out->q8; a.s8 = out->s8;
  a.resid = resid;
  int64_t counters[3] = {0, 0, 0};
  a.info_host = info ? counters : nullptr;
  a.workspace = workspace;
  cudaError_t e = launch_encode(a, static_cast<cudaStream_t>(stream), launcher());
  if (e != cudaSuccess) return cuda_fail(e);
  if (info) {
    info->inexact_rotation_blocks = counters[0];
    info->fp16_unsafe_scales = counters[1];
    info->nonfinite_scores = counters[2];
  }
  return DVSSQ_OK;
}

dvssq_status dvssq_forward_workspace_size(const dvssq_shape *shape, int64_t T, int32_t path,
                                          size_t *bytes) {
  dvssq_status s = check_shape(shape);
  if (s != DVSSQ_OK) return s;
  if (bytes == nullptr || T < 0 || T > (1 << 24)) return DVSSQ_ERR_INVALID_ARG;
  if (path < DVSSQ_PATH_AUTO || path > DVSSQ_PATH_PREFILL) return DVSSQ_ERR_INVALID_ARG;
  const int p = choose_path(path, T);
  if (p == DVSSQ_PATH_DECODE && T > 16) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  *bytes = p == DVSSQ_PATH_DECODE
               ? decode_workspace_bytes(shape->M, shape->K, shape->block, shape->n_sal,
                                        shape->rank, (int)T)
               : prefill_workspace_bytes(shape->M, shape->K, shape->block, shape->n_sal,
                                         shape->rank, (int)T);
  return DVSSQ_OK;
}

dvssq_status dvssq_linear_forward(const dvssq_shape *shape, const dvssq_weights *w,
                                  const void *x, int64_t T, const void *bias, void *y,
                                  int32_t y_dtype, int32_t path, void *workspace,
                                  size_t workspace_bytes, void *stream) {
  dvssq_status s = check_shape(shape);
  if (s != DVSSQ_OK) return s;
  if (w == nullptr || T < 0 || T > (1 << 24)) return DVSSQ_ERR_INVALID_ARG;
  if (y_dtype != DVSSQ_Y_F32 && y_dtype != DVSSQ_Y_BF16) return DVSSQ_ERR_INVALID_ARG;
  if (path < DVSSQ_PATH_AUTO || path > DVSSQ_PATH_PREFILL) return DVSSQ_ERR_INVALID_ARG;
  const int p = choose_path(path, T);
  if (p == DVSSQ_PATH_DECODE && T > 16) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return DVSSQ_OK;
  if (x == nullptr || y == nullptr || workspace == nullptr || w->q4 == nullptr ||
      w->s4 == nullptr || w->s8 == nullptr)
    return DVSSQ_ERR_INVALID_ARG;
  if (shape->n_sal > 0 && (w->sal_idx == nullptr || w->q8 == nullptr)) return DVSSQ_ERR_INVALID_ARG;
  if (shape->rank > 0 && (w->U == nullptr || w->V == nullptr)) return DVSSQ_ERR_INVALID_ARG;
  const void *bufs[] = {x, y, bias, w->q4, w->s4, w->s8, w->sal_idx, w->q8, w->U, w->V};
  for (const void *b : bufs)
    if (b != nullptr && !aligned16(b)) return DVSSQ_ERR_MISALIGNED;
  if (!aligned256(workspace)) return DVSSQ_ERR_MISALIGNED;
  size_t need = 0;
  dvssq_forward_workspace_size(shape, T, path, &need);
  if (workspace_bytes < need) return DVSSQ_ERR_WORKSPACE;
  if ((s = ensure_device()) != DVSSQ_OK) return s;
  ForwardArgs a;
  a.M = shape->M; a.K = shape->K; a.block = shape->block; a.n_sal = shape->n_sal;
  a.rank = shape->rank; a.T = (int)T;
  a.q4 = w->q4; a.s4 = w->s4; a.sal_idx = w->sal_idx; a.q8 = w->q8; a.s8 = w->s8;
  a.U = w->U; a.V = w->V;
  a.x = static_cast<const uint16_t *>(x);
  a.bias = static_cast<const uint16_t *>(bias);
  a.y = y;
  a.y_bf16 = y_dtype == DVSSQ_Y_BF16;
  a.workspace = workspace;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = p == DVSSQ_PATH_DECODE ? launch_decode(a, st, launcher())
                                         : launch_prefill(a, st, launcher());
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

dvssq_status dvssq_materialize(const dvssq_shape *shape, const dvssq_weights *w, void *W_eff,
                               void *stream) {
  dvssq_status s = check_shape(shape);
  if (s != DVSSQ_OK) return s;
  if (w == nullptr || W_eff == nullptr || w->q4 == nullptr || w->s4 == nullptr ||
      w->s8 == nullptr)
    return DVSSQ_ERR_INVALID_ARG;
  if (shape->n_sal > 0 && (w->sal_idx == nullptr || w->q8 == nullptr)) return DVSSQ_ERR_INVALID_ARG;
  if (shape->rank > 0 && (w->U == nullptr || w->V == nullptr)) return DVSSQ_ERR_INVALID_ARG;
  const void *bufs[] = {W_eff, w->q4, w->s4, w->s8, w->sal_idx, w->q8, w->U, w->V};
  for (const void *b : bufs)
    if (b != nullptr && !aligned16(b)) return DVSSQ_ERR_MISALIGNED;
  if ((s = ensure_device()) != DVSSQ_OK) return s;
  MaterializeArgs a;
  a.M = shape->M; a.K = shape->K; a.block = shape->block; a.n_sal = shape->n_sal;
  a.rank = shape->rank;
  a.q4 = w->q4; a.s4 = w->s4; a.sal_idx = w->sal_idx; a.q8 = w->q8; a.s8 = w->s8;
  a.U = w->U; a.V = w->V;
  a.W = static_cast<uint16_t *>(W_eff);
  const cudaError_t e = launch_materialize(a, static_cast<cudaStream_t>(stream), launcher());
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

static dvssq_status lowrank_shape(int32_t M, int32_t K, int32_t rank) {
  if (M < 1 || K < 1 || M > (1 << 24) || K > 65536) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (rank < 8 || rank > 64 || rank % 8 != 0) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (rank + 16 > M || rank + 16 > K) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  return DVSSQ_OK;
}

dvssq_status dvssq_lowrank_workspace_size(int32_t M, int32_t K, int32_t rank, size_t *bytes) {
  if (bytes == nullptr) return DVSSQ_ERR_INVALID_ARG;
  const dvssq_status s = lowrank_shape(M, K, rank);
  if (s != DVSSQ_OK) return s;
  *bytes = lowrank_workspace_bytes(M, K, rank);
  return DVSSQ_OK;
}

dvssq_status dvssq_lowrank(const float *R, int32_t M, int32_t K, int32_t rank, int32_t iters,
                           uint64_t seed, uint16_t *U, uint16_t *V, float *sigma,
                           void *workspace, size_t workspace_bytes, void *stream) {
  dvssq_status s = lowrank_shape(M, K, rank);
  if (s != DVSSQ_OK) return s;
  if (R == nullptr || U == nullptr || V == nullptr || workspace == nullptr || iters < 0 ||
      iters > 64)
    return DVSSQ_ERR_INVALID_ARG;
  const void *bufs[] = {R, U, V, sigma};
  for (const void *b : bufs)
    if (b != nullptr && !aligned16(b)) return DVSSQ_ERR_MISALIGNED;
  if (!aligned256(workspace)) return DVSSQ_ERR_MISALIGNED;
  if (workspace_bytes < lowrank_workspace_bytes(M, K, rank)) return DVSSQ_ERR_WORKSPACE;
  if ((s = ensure_device()) != DVSSQ_OK) return s;
  LowrankArgs a;
  a.R = R; a.M = M; a.K = K; a.rank = rank; a.iters = iters; a.seed = seed;
  a.U = U; a.V = V; a.sigma = sigma; a.workspace = workspace;
  const cudaError_t e = launch_lowrank(a, static_cast<cudaStream_t>(stream), launcher());
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

static dvssq_status bss_shape(const dvssq_attn_shape *s) {
  if (s == nullptr) return DVSSQ_ERR_INVALID_ARG;
  if (s->batch < 1 || s->q_heads < 1 || s->kv_heads < 1 || s->ctx < 1)
    return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (s->q_heads % s->kv_heads != 0) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  const int G = s->q_heads / s->kv_heads;
  const bool ok = (s->head_dim == 256 && (G == 2 || G == 4)) ||
                  (s->head_dim == 128 && (G == 2 || G == 4 || G == 8));
  if (!ok) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if ((long long)s->batch * s->q_heads > 65535 || s->ctx > (1 << 24))
    return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  if (!(s->tau > 0.f) || s->haze != s->haze) return DVSSQ_ERR_INVALID_ARG;
  return DVSSQ_OK;
}

dvssq_status dvssq_bss_attention_workspace_size(const dvssq_attn_shape *shape, size_t *bytes) {
  if (bytes == nullptr) return DVSSQ_ERR_INVALID_ARG;
  const dvssq_status s = bss_shape(shape);
  if (s != DVSSQ_OK) return s;
  *bytes = bss_workspace_bytes(shape->batch, shape->q_heads, shape->ctx, shape->head_dim);
  return DVSSQ_OK;
}

dvssq_status dvssq_bss_attention(const dvssq_attn_shape *shape, const void *q, const void *k,
                                 const void *v, float *out, void *workspace,
                                 size_t workspace_bytes, void *stream) {
  dvssq_status s = bss_shape(shape);
  if (s != DVSSQ_OK) return s;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || workspace == nullptr)
    return DVSSQ_ERR_INVALID_ARG;
  const void *bufs[] = {q, k, v, out};
  for (const void *b : bufs)
    if (!aligned16(b)) return DVSSQ_ERR_MISALIGNED;
  if (!aligned256(workspace)) return DVSSQ_ERR_MISALIGNED;
  if (workspace_bytes < bss_workspace_bytes(shape->batch, shape->q_heads, shape->ctx,
                                            shape->head_dim))
    return DVSSQ_ERR_WORKSPACE;
  if ((s = ensure_device()) != DVSSQ_OK) return s;
  BssArgs a;
  a.q = static_cast<const uint16_t *>(q);
  a.k = static_cast<const uint16_t *>(k);
  a.v = static_cast<const uint16_t *>(v);
  a.out = out;
  a.B = shape->batch; a.Hq = shape->q_heads; a.Hkv = shape->kv_heads; a.L = shape->ctx;
  a.D = shape->head_dim; a.tau = shape->tau; a.haze = shape->haze;
  a.workspace = workspace;
  const cudaError_t e = launch_bss_attention(a, static_cast<cudaStream_t>(stream), launcher());
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

// ------------------------------------------------------------- MLP stack ---
namespace {
// Host-side checks of a stack and its flattening into matrix descriptors.
dvssq_status stack_descs(const dvssq_mlp_layer *layers, int32_t n_layers,
                         std::vector<StackMatDesc> &mats, StackShapeInfo &si) {
  if (layers == nullptr || n_layers < 1 || n_layers > 4096) return DVSSQ_ERR_INVALID_ARG;
  mats.assign((size_t)n_layers * 3, StackMatDesc{});
  for (int l = 0; l < n_layers; ++l)
    for (int mi = 0; mi < 3; ++mi) {
      const dvssq_shape *sh = &layers[l].shape[mi];
      const dvssq_weights *w = &layers[l].w[mi];
      dvssq_status s = check_shape(sh);
      if (s != DVSSQ_OK) return s;
      if (w->q4 == nullptr || w->s4 == nullptr || w->s8 == nullptr) return DVSSQ_ERR_INVALID_ARG;
      if (sh->n_sal > 0 && (w->sal_idx == nullptr || w->q8 == nullptr))
        return DVSSQ_ERR_INVALID_ARG;
      if (sh->rank > 0 && (w->U == nullptr || w->V == nullptr)) return DVSSQ_ERR_INVALID_ARG;
      const void *bufs[] = {w->q4, w->s4, w->s8, w->sal_idx, w->q8, w->U, w->V};
      for (const void *b : bufs)
        if (b != nullptr && !aligned16(b)) return DVSSQ_ERR_MISALIGNED;
      StackMatDesc &m = mats[(size_t)l * 3 + mi];
      m.q4 = w->q4; m.s4 = w->s4; m.sal_idx = w->sal_idx; m.q8 = w->q8; m.s8 = w->s8;
      m.U = w->U; m.V = w->V; m.vh = nullptr;
      m.M = sh->M; m.K = sh->K; m.block = sh->block; m.n_sal = sh->n_sal; m.r = sh->rank;
    }
  if (!stack_shape_info(mats.data(), n_layers, si)) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  return DVSSQ_OK;
}
}  // namespace

dvssq_status dvssq_mlp_stack_workspace_size(const dvssq_mlp_layer *layers, int32_t n_layers,
                                            size_t *bytes) {
  if (bytes == nullptr) return DVSSQ_ERR_INVALID_ARG;
  std::vector<StackMatDesc> mats;
  StackShapeInfo si{};
  dvssq_status s = stack_descs(layers, n_layers, mats, si);
  if (s != DVSSQ_OK) return s;
  *bytes = stack_workspace_bytes(si, n_layers);
  return DVSSQ_OK;
}

dvssq_status dvssq_mlp_stack_plan_query(const dvssq_mlp_layer *layers, int32_t n_layers,
                                        int32_t sm_count, dvssq_mlp_stack_plan *plan) {
  if (plan == nullptr || sm_count < 1) return DVSSQ_ERR_INVALID_ARG;
  std::vector<StackMatDesc> mats;
  StackShapeInfo si{};
  dvssq_status s = stack_descs(layers, n_layers, mats, si);
  if (s != DVSSQ_OK) return s;
  StackPlanInfo pi{};
  if (!stack_plan_info(mats.data(), n_layers, sm_count, pi)) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  plan->ctas = pi.ctas;
  plan->threads = pi.threads;
  plan->ring_slots = pi.slots;
  plan->slot_bytes = pi.slot_bytes;
  plan->rows_per_tile_gate_up = pi.tr_gu;
  plan->rows_per_tile_down = pi.tr_d;
  plan->smem_bytes = pi.smem;
  return DVSSQ_OK;
}

dvssq_status dvssq_mlp_stack_prepare(const dvssq_mlp_layer *layers, int32_t n_layers,
                                     void *workspace, size_t workspace_bytes, void *stream) {
  std::vector<StackMatDesc> mats;
  StackShapeInfo si{};
  dvssq_status s = stack_descs(layers, n_layers, mats, si);
  if (s != DVSSQ_OK) return s;
  if (workspace == nullptr) return DVSSQ_ERR_INVALID_ARG;
  if (!aligned256(workspace)) return DVSSQ_ERR_MISALIGNED;
  if ((s = ensure_device()) != DVSSQ_OK) return s;
  if (workspace_bytes < stack_workspace_bytes(si, n_layers)) return DVSSQ_ERR_WORKSPACE;
  cudaError_t e = stack_prepare(mats.data(), n_layers, si, workspace,
                                static_cast<cudaStream_t>(stream), launcher());
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

dvssq_status dvssq_mlp_stack_forward(const dvssq_mlp_layer *layers, int32_t n_layers,
                                     const void *x, void *y, void *workspace,
                                     size_t workspace_bytes, void *stream) {
  std::vector<StackMatDesc> mats;
  StackShapeInfo si{};
  dvssq_status s = stack_descs(layers, n_layers, mats, si);
  if (s != DVSSQ_OK) return s;
  if (x == nullptr || y == nullptr || workspace == nullptr) return DVSSQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned256(workspace)) return DVSSQ_ERR_MISALIGNED;
  if ((s = ensure_device()) != DVSSQ_OK) return s;
  if (workspace_bytes < stack_workspace_bytes(si, n_layers)) return DVSSQ_ERR_WORKSPACE;
  cudaError_t e = launch_mlp_stack(mats.data(), n_layers, si, x, y, workspace,
                                   static_cast<cudaStream_t>(stream), launcher());
  if (e == cudaErrorNotSupported) return DVSSQ_ERR_UNSUPPORTED_SHAPE;
  return e == cudaSuccess ? DVSSQ_OK : cuda_fail(e);
}

dvssq_status dvssq_device_error(uint32_t *word, int32_t clear) {
  if (word == nullptr) return DVSSQ_ERR_INVALID_ARG;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  if ((e = cudaMemcpyFromSymbol(word, g_dvssq_error, sizeof(uint32_t))) != cudaSuccess)
    return cuda_fail(e);
  if (clear) {
    const uint32_t z = 0;
    if ((e = cudaMemcpyToSymbol(g_dvssq_error, &z, sizeof(uint32_t))) != cudaSuccess)
      return cuda_fail(e);
  }
  return DVSSQ_OK;
}

dvssq_status dvssq_profile_enable(int32_t on) {
  launcher().profiling = on != 0;
  return DVSSQ_OK;
}

dvssq_status dvssq_profile_collect(void) {
  Launcher &L = launcher();
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (ProfileRecord &r : L.pending) {
    cudaError_t e = cudaEventSynchronize(r.stop);
    if (e != cudaSuccess) return cuda_fail(e);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, r.start, r.stop);
    bool found = false;
    for (ProfileTotal &t : g_prof)
      if (strcmp(t.name, r.name) == 0) {
        t.launches += 1;
        t.ms += ms;
        found = true;
        break;
      }
    if (!found) g_prof.push_back({r.name, 1, (double)ms});
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  L.pending.clear();
  return DVSSQ_OK;
}

int32_t dvssq_profile_count(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return (int32_t)g_prof.size();
}

dvssq_status dvssq_profile_get(int32_t i, const char **name, int64_t *launches, double *total_ms) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (i < 0 || i >= (int32_t)g_prof.size()) return DVSSQ_ERR_INVALID_ARG;
  if (name) *name = g_prof[i].name;
  if (launches) *launches = g_prof[i].launches;
  if (total_ms) *total_ms = g_prof[i].ms;
  return DVSSQ_OK;
}

dvssq_status dvssq_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof.clear();
  return DVSSQ_OK;
}

}  // extern "C"
