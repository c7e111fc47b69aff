// Internal interface between the C ABI (dvssq_api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <string>
#include <utility>
#include <vector>

namespace dvssq {

// Largest supported salient set (bounded by the encoder's shared-memory stash).
constexpr int kMaxSalient = 16384;

// ------------------------------------------------------------ launching ---
// Launches kernels with optional programmatic dependent launch and, while
// profiling is enabled, brackets each launch with CUDA events on its stream.
struct ProfileRecord {
  const char *name;
  cudaEvent_t start, stop;
};

class Launcher {
 public:
  bool profiling = false;
  std::vector<ProfileRecord> pending;

  // cluster_y > 0 launches thread-block clusters of (1, cluster_y, 1).
  template <typename... KArgs, typename... Args>
  cudaError_t launch_ex(const char *name, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                        size_t smem, cudaStream_t st, bool pdl, int cluster_y, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl && !profiling) {
      attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[na].val.programmaticStreamSerializationAllowed = 1;
      ++na;
    }
    if (cluster_y > 0) {
      attr[na].id = cudaLaunchAttributeClusterDimension;
      attr[na].val.clusterDim.x = 1;
      attr[na].val.clusterDim.y = (unsigned)cluster_y;
      attr[na].val.clusterDim.z = 1;
      ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    ProfileRecord rec{name, nullptr, nullptr};
    if (profiling) {
      cudaEventCreate(&rec.start);
      cudaEventCreate(&rec.stop);
      cudaEventRecord(rec.start, st);
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    if (profiling) {
      cudaEventRecord(rec.stop, st);
      pending.push_back(rec);
    }
    return e;
  }

  // Cooperative launch: every CTA of the grid is resident at once (the
  // kernel's blocks wait on one another through a grid barrier).
  template <typename... KArgs, typename... Args>
  cudaError_t launch_coop(const char *name, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                          size_t smem, cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ProfileRecord rec{name, nullptr, nullptr};
    if (profiling) {
      cudaEventCreate(&rec.start);
      cudaEventCreate(&rec.stop);
      cudaEventRecord(rec.start, st);
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    if (profiling) {
      cudaEventRecord(rec.stop, st);
      pending.push_back(rec);
    }
    return e;
  }

  template <typename... KArgs, typename... Args>
  cudaError_t launch(const char *name, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                     size_t smem, cudaStream_t st, bool pdl, Args &&...args) {
    return launch_ex(name, kernel, grid, block, smem, st, pdl, 0, std::forward<Args>(args)...);
  }
};

Launcher &launcher();
void set_last_error(const std::string &msg);

// --------------------------------------------------------------- encoder ---
struct EncodeArgs {
  int M, K, block, n_sal;
  const void *W;
  const float *act_scale;
  uint8_t *q4;
  uint16_t *s4;
  int32_t *sal_idx;
  int8_t *q8;
  uint16_t *s8;
  float *resid;
  int64_t *info_host;  // 3 counters or nullptr
  void *workspace;
};
size_t encode_workspace_bytes(int M, int K, int block, int n_sal);
cudaError_t prepare_encode_kernels();
cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t st, Launcher &L);

// ------------------------------------------------------------- MLP stack ---
struct alignas(16) StackMatDesc {   // one packed matrix (device pointers)
  const uint8_t *q4;
  const uint16_t *s4;
  const int32_t *sal_idx;
  const int8_t *q8;
  const uint16_t *s8;
  const uint16_t *U;
  const uint16_t *V;
  const float *vh;              // (V H_K) in FP32 [r][K], in the stack workspace
  int M, K, block, n_sal, r;
};
struct StackLayerDesc {
  StackMatDesc m[3];            // gate, up, down
};
struct StackShapeInfo {
  int H, I, block;
  size_t vh_floats;
};
bool stack_shape_info(const StackMatDesc *mats, int L, StackShapeInfo &si);
size_t stack_workspace_bytes(const StackShapeInfo &si, int L);
// The forward's launch plan for G SMs (host only): false when the stack's
// tiles do not fit the shared-memory ring or G is out of range.
struct StackPlanInfo {
  int ctas, threads, slots, slot_bytes, tr_gu, tr_d, smem;
};
bool stack_plan_info(const StackMatDesc *mats, int L, int G, StackPlanInfo &out);
cudaError_t stack_prepare(StackMatDesc *mats, int L, const StackShapeInfo &si, void *ws,
                          cudaStream_t st, Launcher &Lc);
cudaError_t launch_mlp_stack(const StackMatDesc *mats, int L, const StackShapeInfo &si,
                             const void *x, void *y, void *ws, cudaStream_t st, Launcher &Lc);
cudaError_t prepare_stack_kernels();

// ------------------------------------------------------------ activations -
cudaError_t launch_gelu_mul(const uint16_t *g, const uint16_t *u, uint16_t *h, long long n,
                            cudaStream_t st, Launcher &L);
cudaError_t launch_fwht(const uint16_t *x, float *y, int64_t rows, int cols, int block,
                        cudaStream_t st, Launcher &L);

// ---------------------------------------------------------------- forward -
struct ForwardArgs {
  int M, K, block, n_sal, rank;
  int T;
  const uint8_t *q4;
  const uint16_t *s4;
  const int32_t *sal_idx;
  const int8_t *q8;
  const uint16_t *s8;
  const uint16_t *U;
  const uint16_t *V;
  const uint16_t *x;
  const uint16_t *bias;
  void *y;
  int y_bf16;
  void *workspace;
};

size_t decode_workspace_bytes(int M, int K, int block, int n_sal, int rank, int T);
size_t prefill_workspace_bytes(int M, int K, int block, int n_sal, int rank, int T);
cudaError_t prepare_forward_kernels();
cudaError_t launch_decode(const ForwardArgs &a, cudaStream_t st, Launcher &L);
cudaError_t launch_prefill(const ForwardArgs &a, cudaStream_t st, Launcher &L);

// ------------------------------------------------------------ materialize -
struct MaterializeArgs {
  int M, K, block, n_sal, rank;
  const uint8_t *q4;
  const uint16_t *s4;
  const int32_t *sal_idx;
  const int8_t *q8;
  const uint16_t *s8;
  const uint16_t *U;
  const uint16_t *V;
  uint16_t *W;
};
cudaError_t launch_materialize(const MaterializeArgs &a, cudaStream_t st, Launcher &L);
cudaError_t prepare_materialize_kernels();

// ---------------------------------------------------------------- lowrank -
struct LowrankArgs {
  const float *R;
  int M, K, rank, iters;
  uint64_t seed;
  uint16_t *U, *V;
  float *sigma;
  void *workspace;
};
size_t lowrank_workspace_bytes(int M, int K, int rank);
cudaError_t launch_lowrank(const LowrankArgs &a, cudaStream_t st, Launcher &L);
cudaError_t prepare_lowrank_kernels();

// -------------------------------------------------------- KV-BSS attention -
struct BssArgs {
  const uint16_t *q, *k, *v;
  float *out;
  int B, Hq, Hkv, L, D;
  float tau, haze;
  void *workspace;
};
size_t bss_workspace_bytes(int B, int Hq, int L, int D);
cudaError_t launch_bss_attention(const BssArgs &a, cudaStream_t st, Launcher &L);

// Tensor-map encoder from the driver (resolved once through the runtime).
CUresult encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base,
                        uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                        uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

}  // namespace dvssq
