/*
 * dvssq.h -- C ABI of libdvssq.so, a B200 (sm_100a) implementation of the
 * DV-SSQ compressed linear layer.
 *
 * The method (F-Labs model cards "Spark-X2.5-4B-Hadamard-GSQ", section
 * "Architectural Pillars / 1. DV-SSQ", Tiers A-C, and
 * "MiniCPM5-2B-Hadamard-GSQ", section "Mathematical Foundations" §1-§2):
 *
 *   offline (dvssq_encode):  W_rot = W . H_K, H_K = diag(H_b, ..., H_b), b in
 *     {128, 256}; the top n_sal rotated columns by salience are kept as INT8
 *     with one BF16 scale per row; every other rotated weight is quantised
 *     to symmetric INT4 in groups of 64 contiguous rotated columns with one
 *     BF16 scale per group.
 *   online (dvssq_linear_forward):
 *     y = What4 . (H x) + diag(s8) . Q8 . (H x)_sal + U . (V . (H x)) [+ bias]
 *     with U, V the BF16 truncated-SVD factors of the INT4 residual (A and B
 *     of the MiniCPM card's §2), supplied by the caller.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument named as a buffer is a DEVICE pointer on the
 *   current CUDA device unless documented as host.  Every buffer is owned by
 *   the caller; the library never allocates or frees device memory.  Scratch
 *   memory is the caller's "workspace" (size from the *_workspace_size query).
 * - Matrices are dense and row-major.  BF16 values travel as uint16_t bit
 *   patterns.
 * - Every device buffer must be 16-byte aligned (cudaMalloc gives 256 B);
 *   the workspace must be 256-byte aligned.  Violations return
 *   DVSSQ_ERR_MISALIGNED before any launch.
 * - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t;
 *   NULL is the legacy default stream).  Argument validation happens on the
 *   host before any launch and returns an error status with nothing
 *   launched.  A launch failure returns DVSSQ_ERR_CUDA; dvssq_last_error()
 *   gives the CUDA message.
 * - A workspace must not be shared by calls that may run concurrently.
 * - Kernels never wait without a bound: a wait that runs out sets a device
 *   error word that dvssq_device_error() reads and clears.
 * - Per-device set-up (kernel attributes, constant tables, the address of
 *   the static scratch array) runs on the first call on a device and is kept
 *   for the life of the process: do not use the library across a
 *   cudaDeviceReset of a device it has run on.
 */
#ifndef DVSSQ_H
#define DVSSQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DVSSQ_ABI_VERSION 1

#if defined(__GNUC__)
#define DVSSQ_API __attribute__((visibility("default")))
#else
#define DVSSQ_API
#endif

typedef enum {
  DVSSQ_OK = 0,
  DVSSQ_ERR_INVALID_ARG = 1,      /* NULL pointer, negative size, bad enum      */
  DVSSQ_ERR_UNSUPPORTED_SHAPE = 2,/* shape outside the documented limits        */
  DVSSQ_ERR_MISALIGNED = 3,       /* a buffer is not 16-byte aligned            */
  DVSSQ_ERR_WORKSPACE = 4,        /* workspace smaller than the query's answer  */
  DVSSQ_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed       */
  DVSSQ_ERR_DEVICE = 6            /* current device is not compute capability 10.0 */
} dvssq_status;

/* Shape of one compressed linear layer.
 *   M      out_features (rows of W), 1 <= M <= 2^24
 *   K      in_features, a multiple of `block`, of 64 and of 128, K <= 65536
 *   block  Hadamard block size b: 128 or 256
 *   group  INT4 group size: must be 64
 *   n_sal  number of salient (INT8) columns: 0 <= n_sal <= K, n_sal % 16 == 0;
 *          the method uses n_sal = K / 8 (top 12.5 %)
 *   rank   rank r of the residual factors: 0 <= r <= 64, r % 8 == 0 (the
 *          rows of U travel as 16-byte vectors)                          */
typedef struct {
  int32_t M;
  int32_t K;
  int32_t block;
  int32_t group;
  int32_t n_sal;
  int32_t rank;
} dvssq_shape;

/* The packed layer (all device pointers).  dvssq_encode writes q4, s4,
 * sal_idx, q8 and s8; U and V are inputs supplied by the caller.
 *   q4       uint8 [M][K/2]: INT4 codes of the rotated weights, two's
 *            complement, the even rotated column in the low nibble; codes at
 *            salient columns are 0 (dense layout over all K)
 *   s4       bf16 [M][K/64]: one scale per 64 contiguous rotated columns
 *   sal_idx  int32 [n_sal]: salient rotated-column indices, ascending
 *   q8       int8 [M][n_sal]: INT8 codes; column k belongs to sal_idx[k]
 *   s8       bf16 [M]: one INT8 scale per row
 *   U        bf16 [M][r]: A = U_r sqrt(S_r) of the rotated-domain residual
 *   V        bf16 [r][K]: B = sqrt(S_r) V_r^T, rotated-domain columns        */
typedef struct {
  uint8_t *q4;
  uint16_t *s4;
  int32_t *sal_idx;
  int8_t *q8;
  uint16_t *s8;
  const uint16_t *U;
  const uint16_t *V;
} dvssq_weights;

/* Diagnostics of one encode (host struct, filled when non-NULL). */
typedef struct {
  /* row-blocks whose +-1 Hadamard sums are not provably exact in fp64
     (BF16 exponent spread above 45 - log2(b) bits).  The encoder sums
     these blocks exactly in integers and rounds each sum once, so their
     codes equal an exact-arithmetic encoder's; blocks holding Inf or NaN
     keep the fp64 butterfly's (non-finite) values.  A diagnostic count.  */
  int64_t inexact_rotation_blocks;
  /* INT4 groups with a nonzero scale outside [2^-17, 8188] and rows with a
     nonzero INT8 scale outside [2^-17, 511]: the prefill path stages q*s
     in FP16, which is exact (INT4) or correctly rounded (INT8) only
     inside those ranges                                                   */
  int64_t fp16_unsafe_scales;
  /* NaN or infinite salience scores (from non-finite W or act_scale)      */
  int64_t nonfinite_scores;
} dvssq_encode_info;

/* Output element type of the forward. */
enum { DVSSQ_Y_F32 = 0, DVSSQ_Y_BF16 = 1 };

/* Kernel choice of the forward: AUTO picks the decode GEMV for T <= 16 and
 * the tensor-core GEMM above; the others force one (the GEMV accepts
 * T <= 16, the GEMM any T >= 1).                                          */
enum { DVSSQ_PATH_AUTO = 0, DVSSQ_PATH_DECODE = 1, DVSSQ_PATH_PREFILL = 2 };

/* ABI version of the loaded library (DVSSQ_ABI_VERSION). */
DVSSQ_API int32_t dvssq_abi_version(void);

/* Static description of a status code. */
DVSSQ_API const char *dvssq_status_string(dvssq_status status);

/* Text of the last CUDA error seen by this host thread ("" if none). */
DVSSQ_API const char *dvssq_last_error(void);

/* Blockwise Walsh-Hadamard rotation of activations, x_rot = H_K x
 * (MiniCPM card, Mathematical Foundations §1: X' = X H; Spark card, Tier B:
 * H_K = diag(H_b, ..., H_b)), H_b = S_b / sqrt(b) with S_b Sylvester's
 * +-1 matrix.
 *   x      bf16 [rows][cols]  (device)
 *   y      fp32 [rows][cols]  (device), y[i] = H_K x[i], computed in fp32
 *   rows   >= 0 (0 is a no-op); cols a multiple of block; block 128 or 256
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, DEVICE, CUDA.        */
DVSSQ_API dvssq_status dvssq_fwht(const void *x, float *y, int64_t rows, int32_t cols,
                        int32_t block, void *stream);

/* Gated GELU of a Spark-shaped MLP block, the step between the up and down
 * projections ("Myric/Spark-X2.5-4B-GGUF", "The model": GELU FFN;
 * "Spark-X2.5-4B-ASHQ1-GGUF", "Architecture": ffn_gate / ffn_up /
 * ffn_down).  The pages name the activation only; the gated erf form is this
 * library's reading:
 *   h[i] = RN_bf16( gelu(gate[i]) * up[i] ),  gelu(v) = v/2 (1 + erf(v/sqrt 2))
 * evaluated in FP32.
 *   gate, up  bf16 [n]  (device, caller-owned)
 *   h         bf16 [n]  (device; may alias gate or up)
 *   n         >= 0 (0 is a no-op); all three pointers 16-byte aligned
 * Stream-ordered and asynchronous.
 * Errors: INVALID_ARG, MISALIGNED, DEVICE, CUDA.                            */
DVSSQ_API dvssq_status dvssq_gelu_mul(const void *gate, const void *up, void *h, int64_t n,
                                      void *stream);

/* Bytes of workspace dvssq_encode needs for `shape` (host only; no CUDA). */
DVSSQ_API dvssq_status dvssq_encode_workspace_size(const dvssq_shape *shape, size_t *bytes);

/* Encoder (Spark card, Tiers A and B; MiniCPM card §1-§2):
 *   1. W_rot = W . H_K: each +-1 sum is computed exactly and rounded once
 *      to fp64 (fp64 butterflies where the block's exponent spread makes
 *      them exact, integer sums elsewhere); the scale 1/sqrt(b) is applied
 *      once.
 *   2. score_j = act_scale_j * sqrt(sum_i W_rot[i,j]^2); the sum runs over
 *      rows in chunks of 16 (within a chunk acc = acc + w*w, each operation
 *      rounded), the chunk sums in groups of 8 consecutive chunks (each group
 *      summed from 0 in ascending order), the group sums in ascending order.
 *   3. sal_idx = the n_sal largest scores, ties to the lower index, sorted.
 *   4. INT8 tier per row: s8 = bf16_rn(max_{j in sal} |W_rot| / 127),
 *      q8 = clip(rint(w / s8), -128, 127)  (division as w * (1/s8)).
 *   5. INT4 tier per 64-column group with the salient columns zeroed:
 *      s4 = bf16_rn(absmax / 7), q = clip(rint(w * (1/s4)), -8, 7).
 *   Arguments:
 *   shape      host pointer
 *   W          bf16 [M][K] (device), original (unrotated) weights
 *   act_scale  fp32 [K] (device), activation scale per rotated column
 *   out        host struct of device pointers; q4, s4, sal_idx, q8, s8 are
 *              written (sal_idx/q8 may be NULL when n_sal == 0)
 *   resid      fp32 [M][K] (device) or NULL: R = W_bg - What4 in the
 *              rotated domain, the input of the truncated SVD (Tier C)
 *   info       host struct or NULL; when given the call synchronises
 *              `stream` to fill it
 *   workspace  device scratch of at least dvssq_encode_workspace_size bytes
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, DEVICE, CUDA. */
DVSSQ_API dvssq_status dvssq_encode(const dvssq_shape *shape, const void *W,
                          const float *act_scale, const dvssq_weights *out,
                          float *resid, dvssq_encode_info *info,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace dvssq_linear_forward needs for `shape`, T tokens and
 * `path` (host only). */
DVSSQ_API dvssq_status dvssq_forward_workspace_size(const dvssq_shape *shape, int64_t T,
                                          int32_t path, size_t *bytes);

/* Forward on the packed form (MiniCPM card §2 runtime equation
 * Y = X What^T + (X B^T) A^T, with the Spark card's INT8 salient tier):
 *   y[t][i] = sum_j q4_ij s4_i,j/64 xr[t][j] + s8_i sum_k q8_ik xr[t][sal_k]
 *             + sum_p U_ip (sum_j V_pj xr[t][j]) + bias_i,   xr = H_K x.
 *   shape    host pointer; w: host struct of device pointers (read only)
 *   x        bf16 [T][K] (device); T >= 0 (0 is a no-op)
 *   bias     bf16 [M] (device) or NULL
 *   y        [T][M] (device), fp32 or bf16 by y_dtype (bf16 = round to
 *            nearest even of the fp32 result)
 *   path     DVSSQ_PATH_*
 *   workspace device scratch of at least dvssq_forward_workspace_size bytes
 * Arithmetic:
 *   T <= 2: exact int32 dot products (DP2A) of the codes with xr held as
 *     int16, one FP32 scale per 64 columns (relative step 2^-15; salient
 *     entries one scale per 128-entry chunk); s4/s8 applied in FP32.
 *   3 <= T <= 16: exact FP16 codes times the FP16-rounded xr on tensor cores
 *     with FP32 accumulation; s4/s8 applied in FP32.
 *   T > 16 (GEMM): q*s staged in FP16 (exact for INT4 inside the ranges of
 *     fp16_unsafe_scales) and xr in FP16, accumulating in FP32.
 *   The partial sums are added in a fixed order: results are deterministic.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, DEVICE, CUDA. */
DVSSQ_API dvssq_status dvssq_linear_forward(const dvssq_shape *shape, const dvssq_weights *w,
                                  const void *x, int64_t T, const void *bias,
                                  void *y, int32_t y_dtype, int32_t path,
                                  void *workspace, size_t workspace_bytes,
                                  void *stream);

/* Dense effective weights of a packed layer, in the original (unrotated)
 * domain: the library's counterpart of the Spark card's materialize_weights()
 * ("Spark-X2.5-4B-Hadamard-GSQ", "Quickstart & Inference Guide": the
 * quantised weights materialised as plain BF16):
 *   W_eff = RN_bf16( (What4 + scatter(What8) + U V) . H_K ),
 *   What4[i][j] = q4_ij s4_i,j/64,  What8[i][sal_k] = q8_ik s8_i,
 * so that W_eff x equals the dvssq_linear_forward result up to rounding
 * (H_K is symmetric and H_K^2 = I: MiniCPM card, Mathematical Foundations
 * §1).  Evaluated in FP32 (U V on tensor cores with FP32 accumulation, the
 * Walsh-Hadamard transform in FP32), then rounded once to BF16.
 *   shape, w  as dvssq_linear_forward (w read only; U, V used when rank > 0)
 *   W_eff     bf16 [M][K] (device, caller-owned, 16-byte aligned), written
 * Stream-ordered and asynchronous; no workspace.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, DEVICE, CUDA.        */
DVSSQ_API dvssq_status dvssq_materialize(const dvssq_shape *shape, const dvssq_weights *w,
                                         void *W_eff, void *stream);

/* Bytes of workspace dvssq_lowrank needs (host only). */
DVSSQ_API dvssq_status dvssq_lowrank_workspace_size(int32_t M, int32_t K, int32_t rank,
                                                    size_t *bytes);

/* Rank-r factors of the INT4 residual on the GPU (Spark card, Tier C,
 * "Truncated SVD Low-Rank Residual Compensation": R ~= U_r S_r V_r^T;
 * MiniCPM card, Mathematical Foundations §2: A = U_r sqrt(S_r),
 * B = sqrt(S_r) V_r^T), by randomised subspace iteration: a Gaussian test
 * matrix of p = rank + 16 columns (a counter-based generator keyed by
 * `seed`), `iters` power iterations R R^T with CholeskyQR
 * re-orthonormalisation, then the exact eigen-decomposition (Jacobi, fp64)
 * of the p x p projected Gram matrix.  The truncation error approaches the
 * Eckart-Young optimum sum_{k>r} sigma_k^2 as `iters` grows; the products
 * with R run in FP32, the small problems in fp64, every reduction in a fixed
 * order (deterministic for a given seed).
 *   R      fp32 [M][K] (device): the residual dvssq_encode writes (`resid`)
 *   rank   8 <= rank <= 64, rank % 8 == 0, rank + 16 <= min(M, K)
 *   iters  power iterations, 0..64 (4 is a good default)
 *   U      bf16 [M][rank] (device), written: A = U_r sqrt(S_r)
 *   V      bf16 [rank][K] (device), written: B = sqrt(S_r) V_r^T
 *   sigma  fp32 [rank] (device) or NULL: the estimated singular values
 *   workspace  device scratch of dvssq_lowrank_workspace_size bytes
 * Stream-ordered and asynchronous.  U and V are the inputs U and V of
 * dvssq_weights for the forward.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, DEVICE, CUDA. */
DVSSQ_API dvssq_status dvssq_lowrank(const float *R, int32_t M, int32_t K, int32_t rank,
                                     int32_t iters, uint64_t seed, uint16_t *U, uint16_t *V,
                                     float *sigma, void *workspace, size_t workspace_bytes,
                                     void *stream);

/* KV-BSS attention for decode: one query token per sequence over its whole
 * context ("Spark-X2.5-4B-Hadamard-GSQ", "2. KV-BSS: Key-Value Binding
 * Softmax Sharpening": focus factor scaling and attention haze truncation).
 * Per query head h (KV head h / (q_heads / kv_heads), grouped-query):
 *   s_l = (q_h . k_l) tau / sqrt(head_dim),  m = max_l s_l,
 *   s_l -> -inf where s_l < m - haze  (haze <= 0 disables the truncation),
 *   out_h = softmax(s) . V
 * Logits, the mask decision, the exponentials and the sums are FP32.
 *   batch, q_heads, kv_heads  q_heads % kv_heads == 0; the group size
 *       q_heads / kv_heads is 2, 4 or 8 for head_dim 128 and 2 or 4 for 256
 *   head_dim  128 or 256;  ctx  context length L >= 1
 *   tau, haze the focus factor and the truncation depth (the pages: 1.10, 12)
 */
typedef struct {
  int32_t batch;
  int32_t q_heads;
  int32_t kv_heads;
  int32_t head_dim;
  int32_t ctx;
  float tau;
  float haze;
} dvssq_attn_shape;

/* Bytes of workspace dvssq_bss_attention needs (host only). */
DVSSQ_API dvssq_status dvssq_bss_attention_workspace_size(const dvssq_attn_shape *shape,
                                                          size_t *bytes);

/*   q    bf16 [batch][q_heads][head_dim] (device)
 *   k, v bf16 [batch][kv_heads][ctx][head_dim] (device; the KV cache)
 *   out  fp32 [batch][q_heads][head_dim] (device), written
 *   workspace  device scratch of dvssq_bss_attention_workspace_size bytes
 * Three stream-ordered launches (logits and per-chunk maxima; masked
 * weights and partial P V, skipping V rows masked for every head of a
 * group; the fixed-order merge): results are deterministic.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, DEVICE, CUDA. */
DVSSQ_API dvssq_status dvssq_bss_attention(const dvssq_attn_shape *shape, const void *q,
                                           const void *k, const void *v, float *out,
                                           void *workspace, size_t workspace_bytes,
                                           void *stream);

/* Allocation-free decode forward.  The paper has no counterpart: this entry
 * exists for callers that cannot obtain device memory for a workspace --
 * for example a host program that links only this library and has no device
 * allocator of its own, or a plug-in host that hands its plug-ins fixed input
 * and output buffers and forbids them to allocate.  It computes the same
 * result as dvssq_linear_forward with path DVSSQ_PATH_DECODE (1 <= T <= 16;
 * T == 0 is a no-op), but its scratch lives in a fixed array of
 * DVSSQ_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  It never calls cudaMalloc,
 * cudaFree or any allocating routine.
 *   - Shapes whose decode workspace (dvssq_forward_workspace_size with
 *     DVSSQ_PATH_DECODE) exceeds DVSSQ_STATIC_SCRATCH_BYTES are rejected with
 *     DVSSQ_ERR_WORKSPACE before any launch; dvssq_last_error() then states
 *     the bytes needed and the limit.  T > 16 returns UNSUPPORTED_SHAPE.
 *   - The first call on a device checks the device and looks up the array's
 *     device address (once per device, with that device current, kept until
 *     the process exits); make that first call before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents
 *     (the kernels clear what must start at zero).  Calls that may overlap
 *     on the GPU -- concurrent streams, other host threads -- race on it
 *     and must be serialised by the caller.
 * Other arguments and errors as dvssq_linear_forward.                        */
#define DVSSQ_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)
DVSSQ_API dvssq_status dvssq_linear_forward_static(const dvssq_shape *shape,
                                                   const dvssq_weights *w, const void *x,
                                                   int64_t T, const void *bias, void *y,
                                                   int32_t y_dtype, void *stream);

/* One layer of a stack of gated-GELU MLP blocks ("Myric/Spark-X2.5-4B-GGUF",
 * "The model": GELU FFN; "Spark-X2.5-4B-ASHQ1-GGUF", "Architecture":
 * ffn_gate / ffn_up / ffn_down), each projection in packed DV-SSQ form:
 * shape[0] / w[0] = gate (M = inter, K = hidden), shape[1] / w[1] = up (same
 * shape), shape[2] / w[2] = down (M = hidden, K = inter).  Host struct of
 * device pointers, read only.                                              */
typedef struct {
  dvssq_shape shape[3];
  dvssq_weights w[3];
} dvssq_mlp_layer;

/* Bytes of workspace the MLP-stack calls need for these layers (host only).
 * Supported stacks: every gate/up is inter x hidden and every down hidden x
 * inter with one Hadamard block size; hidden and inter multiples of 512;
 * n_sal a multiple of 32; rank a multiple of 8 and at most 32; and rows
 * small enough that the shared-memory weight ring holds at least two slots
 * (two rows of the down matrix per slot at least: the Spark shapes, hidden
 * 2560 / inter 10240, fit 10 slots of 17.3 KB).  The forward runs one CTA
 * per SM on devices of at most 160 SMs (a B200 has 148).
 * Others return UNSUPPORTED_SHAPE.                                         */
DVSSQ_API dvssq_status dvssq_mlp_stack_workspace_size(const dvssq_mlp_layer *layers,
                                                      int32_t n_layers, size_t *bytes);

/* The launch plan dvssq_mlp_stack_forward uses for these layers on a device
 * of `sm_count` SMs (host only; no device is needed).  The forward runs one
 * CTA per SM; warp 0 of each streams the CTA's weight rows into a ring of
 * shared-memory slots and the other warps compute.
 *   ctas          = sm_count
 *   threads       per CTA
 *   ring_slots    weight-ring slots, each slot_bytes long
 *   rows_per_tile_gate_up, rows_per_tile_down   weight rows per ring slot
 *   smem_bytes    dynamic shared memory per CTA
 * Errors: INVALID_ARG (plan NULL, sm_count < 1, layers as for the workspace
 * query), UNSUPPORTED_SHAPE (the layers, or tiles that leave the ring fewer
 * than two slots, or sm_count above 160), MISALIGNED.                      */
typedef struct {
  int32_t ctas, threads, ring_slots, slot_bytes;
  int32_t rows_per_tile_gate_up, rows_per_tile_down, smem_bytes;
} dvssq_mlp_stack_plan;
DVSSQ_API dvssq_status dvssq_mlp_stack_plan_query(const dvssq_mlp_layer *layers,
                                                  int32_t n_layers, int32_t sm_count,
                                                  dvssq_mlp_stack_plan *plan);

/* Prepares `workspace` for dvssq_mlp_stack_forward on these layers: writes
 * the device table of the layers and, per matrix, (V H_K) in FP32 (the
 * blockwise FWHT of each row of V; H is symmetric).  Synchronises `stream`.
 * Call again whenever a layer's pointers or V change.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, DEVICE, CUDA. */
DVSSQ_API dvssq_status dvssq_mlp_stack_prepare(const dvssq_mlp_layer *layers, int32_t n_layers,
                                               void *workspace, size_t workspace_bytes,
                                               void *stream);

/* One token through the whole stack, in one cooperative launch:
 *   for each layer:  g = RN_bf16(gate(x)), u = RN_bf16(up(x)),
 *                    h = RN_bf16(gelu(g) u)  (as dvssq_gelu_mul),
 *                    x = RN_bf16(down(h));
 *   y = x after the last layer.
 * Each projection is the dvssq_linear_forward equation without bias, with
 * the rank-r input t = V (H x) formed as (V H) x.  Rows are computed as exact
 * int32 dot products of the codes with int16 activations (one scale per 64
 * rotated columns, one per 32 salient entries), scaled in FP32.
 *   layers, n_layers  as given to dvssq_mlp_stack_prepare for `workspace`
 *   x  bf16 [hidden] (device);  y  bf16 [hidden] (device; may alias x)
 * Stream-ordered and asynchronous.  A wait that runs out sets the device
 * error word (dvssq_device_error) and the call's output is then undefined.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, DEVICE, CUDA. */
DVSSQ_API dvssq_status dvssq_mlp_stack_forward(const dvssq_mlp_layer *layers, int32_t n_layers,
                                               const void *x, void *y, void *workspace,
                                               size_t workspace_bytes, void *stream);

/* Reads (and clears when `clear` != 0) the device error word of the current
 * device; synchronises the device.  0 means no kernel gave up a wait; bit 0:
 * an mbarrier wait ran out, bit 1: a tensor-memory accumulator wait, bit 2:
 * a kernel saw an unsupported shape, bit 3: a grid-barrier wait.          */
DVSSQ_API dvssq_status dvssq_device_error(uint32_t *word, int32_t clear);

/* Wait limit of every bounded wait in the library's kernels, in SM clock
 * cycles (default 4e9, about 2 s); cycles <= 0 restores the default.  Not
 * part of the method: it lets a test shorten the limit so that a wait runs
 * out quickly.  Applies to the current device; synchronises it.
 * Errors: DEVICE, CUDA.                                                    */
DVSSQ_API dvssq_status dvssq_set_wait_limit(int64_t cycles);

/* Bounded-wait self-test (not part of the method): launches one warp that
 * waits, through the kernels' own bounded-wait helpers, on something that
 * is never signalled -- which = 0: an mbarrier expecting an arrival that
 * never comes; which = 1: a grid-barrier counter nobody increments.  The
 * wait gives up after the wait limit, sets bit 0 (mbarrier) or bit 3 (grid
 * barrier) of the device error word, and the kernel returns; nothing
 * faults, and the context stays usable.  Stream-ordered.
 * Errors: INVALID_ARG, DEVICE, CUDA.                                       */
DVSSQ_API dvssq_status dvssq_selftest_wait(int32_t which, void *stream);

/* Per-kernel device timing.  While enabled, every launch is bracketed by
 * CUDA events on its own stream (and launched without programmatic
 * dependent launch).  dvssq_profile_collect synchronises those events and
 * adds their elapsed times to per-kernel totals; dvssq_profile_get reads
 * entry i (i < dvssq_profile_count()): its kernel name (static string),
 * launch count and total milliseconds.  dvssq_profile_reset clears them. */
DVSSQ_API dvssq_status dvssq_profile_enable(int32_t on);
DVSSQ_API dvssq_status dvssq_profile_collect(void);
DVSSQ_API int32_t dvssq_profile_count(void);
DVSSQ_API dvssq_status dvssq_profile_get(int32_t i, const char **name, int64_t *launches,
                               double *total_ms);
DVSSQ_API dvssq_status dvssq_profile_reset(void);

#ifdef __cplusplus
}
#endif

#endif /* DVSSQ_H */
