/*
 * svdq.h -- C ABI of the SVDQuant W4A4 + low-rank linear layer for B200 (sm_100a).
 *
 * The layer (SVDQuant summary page, hoonably.github.io/blog/svdquant,
 * section 4.2 "SVDQuant: absorbing outliers via low-rank branch", eq. for XW):
 *
 *     Y = act( Q(X diag(lambda)^-1) Q(R) + (X diag(lambda)^-1 L1) L2 + b ),
 *     R = diag(lambda) W^T - L1 L2,
 *
 * with W in nn.Linear layout [N, K], L1 [K, r] and L2 [r, N] the top-r SVD
 * factors of the smoothed weight (L1 = U_r Sigma_r, L2 = V_r^T, same section),
 * Q the NVFP4 quantizer (E2M1 elements, one E4M3 scale per 16 consecutive
 * elements along K, one float32 scale per tensor; the page's quantizer of
 * section 3 "Quantization preliminary" with q_max = 6, applied per block),
 * and act either the identity or tanh-GELU.
 *
 * Conventions for every entry point:
 *   - Return value: svdq_status.  No entry point aborts, exits or traps; on
 *     failure a message is left in svdq_last_error() (thread local).
 *   - Device memory is owned by the caller (allocate it with PyTorch, cudaMalloc,
 *     a pool...).  The library never allocates device memory.  The layer handle
 *     owns host memory only.
 *   - Streams are cudaStream_t values passed as void*; NULL is the legacy
 *     default stream.  Launching entry points are asynchronous and stream
 *     ordered unless stated otherwise.
 *   - svdq_quantize_act and svdq_w4a4_linear(_qkv_norm_rope) launch with programmatic
 *     dependent launch: their prologue may overlap the previous kernel in the
 *     stream, but they touch no global memory before that kernel has completed
 *     (griddepcontrol.wait), so ordinary stream order holds for the caller.
 *     They also let the next kernel in the stream start early; only a kernel
 *     that was itself launched with programmatic stream serialization can, and
 *     it must wait in the same way before reading their outputs.
 *   - One activation buffer serves one call at a time: two launches that use
 *     the same buffer must be ordered (same stream or events).
 *   - bf16 arrays are passed as raw 16-bit patterns (uint16_t / void*).
 *   - Inputs must be finite; NaN/Inf inputs give unspecified (but memory-safe)
 *     results.
 *   - Shapes: K and N multiples of 64, rank and LoRA rank multiples of 16,
 *     rank capacity <= 256, any M >= 1 (partial tiles are masked).
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SVDQ_ABI_VERSION 1

#if defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARGUMENT = 1,  /* null pointer, M < 1, bad enum value        */
  SVDQ_ERR_UNSUPPORTED_SHAPE = 2, /* K or N % 64, rank % 16, rank > capacity ... */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 3,/* not an sm_100 device (the pages: a capability
                                     check must fail loudly rather than return
                                     wrong output -- Diffusers/Nunchaku page,
                                     "kernel variants per GPU generation")       */
  SVDQ_ERR_BUFFER_TOO_SMALL = 4,  /* a caller buffer is smaller than required    */
  SVDQ_ERR_CUDA = 5,              /* a CUDA runtime call failed                  */
  SVDQ_ERR_TIMEOUT = 6,           /* a kernel's bounded wait ran out (see poll)  */
  SVDQ_ERR_INTERNAL = 7,          /* a library invariant was violated            */
  SVDQ_ERR_HOST_ALLOC = 8         /* host memory allocation failed               */
} svdq_status;

typedef struct svdq_layer svdq_layer; /* opaque host handle of one prepared layer */

/*
 * 4-bit formats (the Diffusers/Nunchaku page: the svdq_w4a4 kernel family has
 * NVFP4 and INT4 variants, chosen by --precision nvfp4|int4 at quantization):
 *   SVDQ_FMT_NVFP4: E2M1 codes with an E4M3 scale per 16 elements along K and a
 *     float32 tensor scale (g_a for X_hat, g_w for R);
 *   SVDQ_FMT_INT4: codes -7..7 with a bf16 scale per 64 elements along K,
 *     s = bf16(amax / 7) (the summary page's quantizer round(X / s),
 *     s = max|X| / q_max, with q_max = 7); no tensor scale.  tcgen05 has no
 *     4-bit integer MMA, so kernel 2 widens the codes to f16 values q s 2^e in
 *     shared memory and runs the f16 MMA; e is a per-layer power of two (e_a
 *     for X_hat from the calibration maximum, e_w for R), reported as
 *     g_a = 2^-e_a and g_w = 2^-e_w.  Inputs whose |X_hat| exceeds 32 times the
 *     calibration maximum saturate in that operand (a scale above 9352, the
 *     largest f16 value whose sevenfold stays finite, after the prescale is
 *     clamped there).  The fused QKV and MLP entry points
 *     take NVFP4 layers only.
 */
enum { SVDQ_FMT_NVFP4 = 1, SVDQ_FMT_INT4 = 2 };
enum { SVDQ_PREPARE_KEEP_R = 1 /* keep float32 R in the handle for SVDQ_EXPORT_R */ };
enum { SVDQ_EPI_NONE = 0, SVDQ_EPI_GELU_TANH = 1 };

/*
 * Offline preparation parameters (the quantize step of the Diffusers page's
 * calibrate / quantize / package workflow; its "--precision nvfp4" and
 * "--rank" flags are `format` and `rank`).
 */
typedef struct svdq_prepare_desc {
  int64_t K;               /* in features, multiple of 64                          */
  int64_t N;               /* out features, multiple of 64 (a fused QKV layer is
                              W_q, W_k, W_v concatenated along N in that order)    */
  int32_t rank;            /* r of the low-rank branch, multiple of 16, may be 0   */
  int32_t rank_capacity;   /* >= rank, multiple of 16, <= 256: room for LoRA ranks */
  int32_t format;          /* SVDQ_FMT_NVFP4 or SVDQ_FMT_INT4                      */
  int32_t num_threads;     /* host threads for preparation; 0 = all cores          */
  int32_t flags;           /* SVDQ_PREPARE_* bits                                  */
  const uint16_t* W;       /* host bf16 [N, K] row-major (nn.Linear weight)        */
  const uint16_t* bias;    /* host bf16 [N], or NULL                               */
  const float* act_amax;   /* host float [K]: max_i |X_ij| over calibration rows
                              (see svdq_calibrate_amax); sets lambda and the static
                              activation tensor scale.  Finite and >= 0, else
                              SVDQ_ERR_INVALID_ARGUMENT                             */
  const uint16_t* L1;      /* optional host bf16 [K, rank]: use these low-rank
                              factors (e.g. from a checkpoint) instead of the
                              library's SVD; NULL = compute them                   */
  const uint16_t* L2;      /* optional host bf16 [rank, N]; both or neither        */
  uint64_t svd_seed;       /* seed of the randomized SVD's test matrix             */
  int32_t svd_power_iters; /* subspace iterations, 0 = default (8)                 */
  int32_t svd_oversample;  /* extra columns of the sketch, 0 = default (16)        */
} svdq_prepare_desc;

/* Library version of this header (SVDQ_ABI_VERSION). */
SVDQ_API int svdq_abi_version(void);

/* Thread-local message of the last failure in this thread ("" if none). */
SVDQ_API const char* svdq_last_error(void);

/*
 * Calibration statistic: amax[j] = max(amax[j], max_i |X_ij|) over the M rows
 * of a host bf16 [M, K] batch.  Initialise amax to zeros before the first
 * batch.  Host only; no CUDA call.
 */
SVDQ_API svdq_status svdq_calibrate_amax(const uint16_t* X, int64_t M, int64_t K, float* amax);

/*
 * Bytes of device memory a layer with this descriptor needs (weights, scales,
 * smoothing factors, low-rank factors at rank_capacity, bias, status word).
 * Returns 0 if the descriptor is invalid (svdq_last_error says why).
 */
SVDQ_API size_t svdq_layer_device_bytes(const svdq_prepare_desc* d);

/*
 * Host half of the preparation, no CUDA call (usable without a GPU):
 *   lambda_j = sqrt(act_amax_j / max_n |W_nj|) (1 where either is 0), float32;
 *   W_hat^T = diag(lambda) W^T; top-r factors by randomized subspace iteration
 *   (Halko, Martinsson & Tropp 2011) + one-sided Jacobi SVD, rounded to bf16
 *   (or the caller's L1/L2); R = W_hat^T - L1 L2 in float64; NVFP4 of R^T with
 *   g_w = max|R| / 2688; static activation scale g_a from act_amax.
 * (SVDQuant summary page, section 4.2.)  The result is packed into the
 * device image (tiled, swizzled layouts of the kernels) held by the handle.
 * *out must be released with svdq_layer_destroy.
 */
SVDQ_API svdq_status svdq_prepare_host(const svdq_prepare_desc* d, svdq_layer** out);

/*
 * Device half: checks the current device is sm_100 (SVDQ_ERR_UNSUPPORTED_DEVICE
 * otherwise), copies the image into dev_buf (>= svdq_layer_device_bytes,
 * 256-byte aligned) on stream s and synchronizes s.  The handle remembers
 * dev_buf and the current device; dev_buf must outlive the handle's use.
 */
SVDQ_API svdq_status svdq_layer_upload(svdq_layer* layer, void* dev_buf, size_t dev_buf_bytes, void* stream);

/* svdq_prepare_host followed by svdq_layer_upload. */
SVDQ_API svdq_status svdq_prepare_weights(const svdq_prepare_desc* d, void* dev_buf, size_t dev_buf_bytes,
                                 svdq_layer** out, void* stream);

/*
 * Bytes of the per-call activation buffer for M tokens: NVFP4 codes and block
 * scales of X_hat in the GEMM's tiled layout, the bf16 down-projection
 * lr' = (X_hat L1) / (g_a g_w) for rank_capacity ranks.  Host only.
 */
SVDQ_API svdq_status svdq_act_buffer_bytes(const svdq_layer* layer, int64_t M, size_t* bytes);

/*
 * Kernel 1 (Nunchaku fusion of the down projection into the quantizer,
 * SVDQuant summary page section 4.3 / Figure 6(b)).  One pass over X:
 *   x_hat = bf16(x / lambda); per 16 elements along K: E4M3 block scale,
 *   E2M1 codes (INT4 layer: per 64 elements a bf16 scale and codes -7..7);
 *   lr' = bf16((x_hat L1) / (g_a g_w)) on the tensor cores.
 * X: device bf16 [M, K] row-major, 16-byte aligned, row stride K.
 * act_buf: device, >= svdq_act_buffer_bytes(M) bytes, 256-byte aligned.
 */
SVDQ_API svdq_status svdq_quantize_act(const svdq_layer* layer, const void* X, int64_t M, void* act_buf,
                              size_t act_buf_bytes, void* stream);

/*
 * Kernel 2 (Nunchaku fusion of the up projection into the 4-bit GEMM, same
 * section): Y = act(g_a g_w (Q(X_hat) Q(R) + lr' L2) + b) with the FP4
 * block-scaled MMA and the bf16 up projection accumulating into the same
 * tensor-memory tile (INT4 layer: the f16 MMA on the widened codes, see
 * SVDQ_FMT_INT4).
 * act_buf: the buffer svdq_quantize_act filled for the same M, through this
 *   handle, after its last svdq_lora_swap.  The handle notes the last 64 act_bufs
 *   it filled; one of those filled before a later swap holds lr' columns of the
 *   replaced factors, and is refused with SVDQ_ERR_INVALID_ARGUMENT (quantize X
 *   again).  A buffer filled through another handle is not checked.
 * Y: device bf16 [M, N] row-major, 32-byte aligned.
 * epilogue: SVDQ_EPI_NONE or SVDQ_EPI_GELU_TANH (bias is added first).
 */
SVDQ_API svdq_status svdq_w4a4_linear(const svdq_layer* layer, const void* act_buf, size_t act_buf_bytes,
                             int64_t M, void* Y, int epilogue, void* stream);

/*
 * Kernel 2 for a fused Q | K | V projection (Diffusers/Nunchaku page,
 * fused-QKV section: to_q, to_k, to_v concatenated along the output dimension
 * in that order, and the projection, the Q/K normalization and the rotary
 * embedding handed to one fused operator).  The layer's output
 * y = bf16(g_a g_w (Q(X_hat) Q(R) + lr' L2) + b), as svdq_w4a4_linear with
 * SVDQ_EPI_NONE returns it, is split along N into Q, K and V of N / 3 columns,
 * and those into heads of head_dim columns.  For every Q and K head of a row:
 *   z = y / sqrt(mean(y^2) + eps) * w      (w = norm_q for Q, norm_k for K)
 *   (z[2i], z[2i+1]) -> (z[2i] c - z[2i+1] s, z[2i+1] c + z[2i] s)
 * with (c, s) the rotary angle of pair i of the row, in float32, rounded to
 * bf16 once at the end.  V is written as y.  The page names the operator but
 * not its arithmetic: the norm and the rotation above are the plain RMSNorm
 * and rotary embedding.
 * head_dim: 128 (SVDQ_ERR_UNSUPPORTED_SHAPE otherwise; N / 3 must be a
 *   multiple of it).
 * norm_q, norm_k: device bf16 [head_dim], 16-byte aligned.
 * rope_packed: device, >= svdq_rope_packed_bytes(M) bytes, 16-byte aligned,
 *   written by svdq_rope_pack from the [M][head_dim / 2][2] table; row m of Y
 *   uses row m of the table.  One packed table serves every layer and call
 *   with the same rows.
 * eps: finite, >= 0 (FLUX uses 1e-6).  With eps = 0 an all-zero Q or K head
 *   is 0 / 0 and comes out NaN, as the formula gives.
 * act_buf, M, Y, stream: as svdq_w4a4_linear.
 */
SVDQ_API svdq_status svdq_w4a4_linear_qkv_norm_rope(const svdq_layer* layer, const void* act_buf,
                                           size_t act_buf_bytes, int64_t M, void* Y, const void* norm_q,
                                           const void* norm_k, const void* rope_packed,
                                           size_t rope_packed_bytes, int32_t head_dim, float eps,
                                           void* stream);

/*
 * The fused MLP pair (Diffusers/Nunchaku page, the kernel-family list: the
 * fused GELU/MLP path).  Runs fc1's kernel 2 on act1, and instead of writing
 * fc1's output y = bf16(act(g_a g_w (Q(X_hat) Q(R) + lr' L2) + b)) it turns each
 * row of it straight into fc2's activation buffer: x_hat2 = bf16(y / lambda2)
 * with fc2's smoothing factors, its NVFP4 codes and E4M3 block scales under
 * fc2's static g_a, and lr'2 = bf16((x_hat2 L1_2) / (g_a2 g_w2)) -- exactly what
 * svdq_quantize_act(fc2, y) computes from the bf16 y, without y ever reaching
 * memory.  Then svdq_w4a4_linear(fc2, act2, ...) finishes the pair.
 * fc2's K must equal fc1's N.  act1: filled by svdq_quantize_act(fc1) for the
 * same M.  act2: >= svdq_act_buffer_bytes(fc2, M) bytes, 256-byte aligned.
 * workspace: device, 16-byte aligned, >= svdq_mlp_workspace_bytes bytes (0 when
 *   fc2 has no ranks): float partials of x_hat2 L1_2, one per 256 of fc1's
 *   outputs, which a second kernel on the same stream sums in a fixed order.
 *   It is scratch: reused by the next call, caller-owned.
 * epilogue: SVDQ_EPI_GELU_TANH (the MLP's activation) or SVDQ_EPI_NONE.
 * Stream ordered; both layers on the current device.
 */
SVDQ_API svdq_status svdq_mlp_workspace_bytes(const svdq_layer* fc1, const svdq_layer* fc2, int64_t M,
                                              size_t* bytes);
SVDQ_API svdq_status svdq_w4a4_linear_mlp(const svdq_layer* fc1, const void* act1, size_t act1_bytes, int64_t M,
                                          const svdq_layer* fc2, void* act2, size_t act2_bytes, void* workspace,
                                          size_t workspace_bytes, int epilogue, void* stream);

/*
 * svdq_w4a4_linear_mlp without a workspace argument, for callers that cannot
 * allocate device memory: code that runs where a cudaMalloc is not allowed or
 * not wanted (an allocator that owns all of the GPU's memory, a plugin handed
 * only its inputs and outputs, a framework that forbids allocation inside its
 * callbacks).  The scratch partials live in one area of
 * SVDQ_MLP_STATIC_SCRATCH_BYTES inside the library (a __device__ array): every
 * GPU that loads the library holds it until the process exits.  The pages have
 * no counterpart; it computes exactly what svdq_w4a4_linear_mlp computes.
 * The first call on a device looks the area's address up (with that device
 * current); make that first call before any stream capture.  Every call on a
 * device shares the one area: calls whose kernels overlap on the GPU (other
 * streams, other threads) race on it and give wrong results.  Nothing in the
 * area needs to start at zero (each call overwrites every partial it reads);
 * it keeps the last call's contents.  A pair whose partials need more than the
 * area holds (svdq_mlp_workspace_bytes) is refused with
 * SVDQ_ERR_UNSUPPORTED_SHAPE before anything is launched.  Allocates nothing.
 */
#define SVDQ_MLP_STATIC_SCRATCH_BYTES (32u << 20)
SVDQ_API svdq_status svdq_w4a4_linear_mlp_static(const svdq_layer* fc1, const void* act1, size_t act1_bytes,
                                                 int64_t M, const svdq_layer* fc2, void* act2, size_t act2_bytes,
                                                 int epilogue, void* stream);

/* Bytes of the packed rotary table for M rows (head_dim 128).  Host only. */
SVDQ_API svdq_status svdq_rope_packed_bytes(int64_t M, int32_t head_dim, size_t* bytes);

/*
 * Pack a rotary table for svdq_w4a4_linear_qkv_norm_rope: rope is device float
 * [M][head_dim / 2][2] = (cos, sin) of each row's pairs (16-byte aligned); the
 * packed copy puts the same values in the order the epilogue's threads (one
 * output row each) read them: row tiles of 128, then chunks of 2 pairs, then
 * rows.  Stream ordered.  SVDQ_ERR_BUFFER_TOO_SMALL if packed_bytes is short.
 */
SVDQ_API svdq_status svdq_rope_pack(const void* rope, int64_t M, int32_t head_dim, void* packed,
                                    size_t packed_bytes, void* stream);

/*
 * Attach a LoRA adapter to the low-rank branch without touching R (abstract of
 * arXiv 2411.05007: off-the-shelf LoRAs without re-quantization).  Device
 * bf16 A [K, r_e] and B [r_e, N] (row-major, 2-byte aligned); the layer computes
 * Y += scale X A B by storing L1' = [L1 | bf16(lambda A scale)], L2' = [L2 ; B].
 * r_e = 0 detaches the current adapter.  rank + r_e <= rank_capacity.
 * Stream ordered, no host synchronization; calls on `layer` issued after this
 * one (on any stream ordered after s) see the new rank.  Activation buffers
 * filled before the swap must be filled again before the next linear call (the
 * linear calls refuse them).  Not thread safe against concurrent calls on the
 * same handle.
 */
SVDQ_API svdq_status svdq_lora_swap(svdq_layer* layer, const void* A, const void* B, int32_t r_e, float scale,
                           void* stream);

/* What svdq_layer_export can copy out (logical, unswizzled layouts). */
enum {
  SVDQ_EXPORT_LAMBDA = 1,     /* float [K]                                        */
  SVDQ_EXPORT_INV_LAMBDA = 2, /* float [K]                                        */
  SVDQ_EXPORT_L1 = 3,         /* bf16 [K, rank] (base factors)                    */
  SVDQ_EXPORT_L2 = 4,         /* bf16 [rank, N]                                   */
  SVDQ_EXPORT_R = 5,          /* float [K, N] = float32(R)                        */
  SVDQ_EXPORT_W_CODES = 6,    /* uint8 [N, K/2] E2M1 codes of R^T, element 2i in
                                 the low nibble (INT4: two's-complement codes)    */
  SVDQ_EXPORT_W_SCALES = 7,   /* uint8 [N, K/16] E4M3 block scales (INT4: bf16
                                 bits [N, K/64], N K / 32 bytes)                  */
  SVDQ_EXPORT_SIGMA = 8,      /* double [rank] singular values (library SVD only) */
  SVDQ_EXPORT_SCALARS = 9,    /* float [4]: g_a, g_w, alpha = g_a g_w, 1/alpha    */
  SVDQ_EXPORT_RESID_NORM = 10 /* double [2]: ||W_hat^T - L1 L2||_F with float64
                                 factors, and with the bf16 factors               */
};

/* Copy one prepared array from the handle's host image into host_dst. */
SVDQ_API svdq_status svdq_layer_export(const svdq_layer* layer, int what, void* host_dst, size_t bytes);

/*
 * Unpack a host copy of an activation buffer (M rows) into logical layouts:
 * codes uint8 [M, K/2], scales uint8 [M, K/16], lr bf16 [M, rank_total]
 * (rank_total = rank + attached LoRA rank).  Any output may be NULL.  For an
 * INT4 layer the codes are two's-complement nibbles and `scales` receives bf16
 * bits [M, K/64] (M K / 32 bytes).
 */
SVDQ_API svdq_status svdq_act_unpack(const svdq_layer* layer, int64_t M, const void* act_host, size_t bytes,
                            uint8_t* codes, uint8_t* scales, uint16_t* lr);

/*
 * The prepared layer as one flat, versioned host blob: what a checkpoint
 * stores in place of W (the Diffusers/Nunchaku page, the sections on loading a
 * quantized checkpoint with its quantization_config: a quantized model is
 * saved and loaded without quantizing again).  The blob holds the device image
 * in its base state (rank r, no adapter: an attached LoRA is not saved), the
 * smoothing factors, the bf16 factors L1 and L2, the scalars and, when the
 * library's SVD made the factors, the singular values; a 64-bit FNV-1a
 * checksum covers everything after its 128-byte header.  Host only.
 * svdq_layer_serialize: with host_dst NULL, only *bytes_needed is set; else
 *   writes the blob (SVDQ_ERR_BUFFER_TOO_SMALL if bytes is short).  R itself
 *   (SVDQ_EXPORT_R) is not saved.
 * svdq_layer_import: a new host handle from a blob (validated: magic, version,
 *   shape, section sizes, checksum; SVDQ_ERR_INVALID_ARGUMENT or
 *   SVDQ_ERR_UNSUPPORTED_SHAPE otherwise); upload it with svdq_layer_upload.
 *   The caller keeps ownership of the blob and may free it on return.
 */
SVDQ_API svdq_status svdq_layer_serialize(const svdq_layer* layer, void* host_dst, size_t bytes,
                                          size_t* bytes_needed);
SVDQ_API svdq_status svdq_layer_import(const void* blob, size_t bytes, svdq_layer** out);

typedef struct svdq_layer_info {
  int64_t K, N;
  int32_t rank, rank_total, rank_capacity, format;
  float g_a, g_w, alpha;
  size_t device_bytes;
  void* dev_buf;  /* NULL before upload */
  int32_t device; /* CUDA ordinal, -1 before upload */
} svdq_layer_info;

SVDQ_API svdq_status svdq_get_layer_info(const svdq_layer* layer, svdq_layer_info* info);

/*
 * Read and clear the layer's device status word (synchronizes `stream`).
 * SVDQ_ERR_TIMEOUT if any kernel of this layer gave up a bounded wait since the
 * last poll (its outputs are then invalid), SVDQ_OK otherwise.
 */
SVDQ_API svdq_status svdq_poll_status(const svdq_layer* layer, void* stream);

/* Free the handle's host memory (the caller frees dev_buf). NULL is a no-op. */
SVDQ_API void svdq_layer_destroy(svdq_layer* layer);

/*
 * Host-only copy of a prepared layer: the packed image in its base state
 * (rank r, no adapter), lambda, the factors and the scalars, not bound to any
 * device buffer.  Upload the copy to another buffer or another GPU (one
 * replica per GPU, or several copies on one GPU) without repeating the
 * preparation.  Attached adapters are not copied.  *out must be released
 * with svdq_layer_destroy.  No CUDA call.
 */
SVDQ_API svdq_status svdq_layer_clone(const svdq_layer* layer, svdq_layer** out);

/*
 * The W4A16 layer (Diffusers/Nunchaku page: the awq_w4a16 kernel family, 4-bit
 * weights with 16-bit activations, for the memory-bound adaptive-norm and
 * modulation projections; SVDQuant summary page, section 2 "AWQ": protect the
 * weights by shifting scale onto the activations):
 *
 *     Y = g f16(X diag(s)^-1) deq(Q(W diag(s)))^T + b
 *
 * Q is the NVFP4 quantizer of the W4A4 layer (E2M1 codes, an E4M3 scale per 16
 * weights along K, tensor scale g = max|W diag(s)| / 2688); s is one positive
 * activation-aware scale per input channel (the pages give no rule for it:
 * it is an input, 1 when NULL).  The activations are divided by s in float32
 * and rounded once to f16 (saturating at +-65504), as X_hat is rounded to a
 * 16-bit operand in the W4A4 layer; products are exact, sums float32, Y bf16.
 * The path is built for the small batches of the modulation layers.
 */
typedef struct svdq_w4a16 svdq_w4a16;

typedef struct svdq_w4a16_desc {
  int64_t K;          /* input features, multiple of 64, <= 12288 */
  int64_t N;          /* output features, >= 1 */
  const void* W;      /* host bf16 [N, K] (nn.Linear layout) */
  const float* s;     /* host float [K] activation-aware scales (> 0), or NULL */
  const void* bias;   /* host bf16 [N], or NULL */
} svdq_w4a16_desc;

/* Bytes of the device image (the caller allocates it, 256-byte aligned). 0 on a bad descriptor. */
SVDQ_API size_t svdq_w4a16_device_bytes(const svdq_w4a16_desc* d);

/* Host half: quantize W diag(s) into a new handle (no CUDA call). */
SVDQ_API svdq_status svdq_w4a16_prepare_host(const svdq_w4a16_desc* d, svdq_w4a16** out);

/* Device half: copy the image into dev_buf on `stream` and synchronize it. */
SVDQ_API svdq_status svdq_w4a16_upload(svdq_w4a16* layer, void* dev_buf, size_t dev_buf_bytes, void* stream);

/*
 * Y = g f16(X diag(s)^-1) deq^T + b.  X: device bf16 [M, K] row-major,
 * 16-byte aligned; Y: device bf16 [M, N] row-major, 2-byte aligned; any M >= 1
 * (rows go 8 at a time, one launch each, stream ordered).  Inside a CTA the
 * weight ring's waits are bounded: a wait that gives up sets the status word
 * of the layer's image and the CTA drains its copies and exits (its output
 * rows are then unwritten); svdq_w4a16_poll_status reports it.
 * Range: the divided activation x / s is rounded to f16, not kept as bf16.
 * Magnitudes above 65504 saturate to +-65504 and magnitudes below 2^-14 lose
 * bits (f16 subnormals, zero below 2^-25); between them f16 keeps 3 more bits
 * than bf16.  Inputs with |x / s| outside [2^-14, 65504] are therefore not
 * represented as a bf16 operand would represent them.
 */
SVDQ_API svdq_status svdq_w4a16_linear(const svdq_w4a16* layer, const void* X, int64_t M, void* Y, void* stream);

/*
 * Copy from the handle's host image: SVDQ_EXPORT_W_CODES uint8 [N, K/2] (E2M1,
 * element 2i in the low nibble), SVDQ_EXPORT_W_SCALES uint8 [N, K/16] (E4M3),
 * SVDQ_EXPORT_INV_LAMBDA float [K] (1/s), SVDQ_EXPORT_SCALARS float [1] (g).
 */
SVDQ_API svdq_status svdq_w4a16_export(const svdq_w4a16* layer, int what, void* host_dst, size_t bytes);

/*
 * Reads (and clears) the status word of an uploaded W4A16 layer on `stream`
 * (synchronizing it): SVDQ_OK, or SVDQ_ERR_TIMEOUT if a kernel gave up a
 * bounded wait since the last poll.
 */
SVDQ_API svdq_status svdq_w4a16_poll_status(const svdq_w4a16* layer, void* stream);

/* Free the handle's host memory (the caller frees dev_buf). NULL is a no-op. */
SVDQ_API void svdq_w4a16_destroy(svdq_w4a16* layer);

/*
 * Test hooks.
 * svdq_test_override_device_arch: pretend the device reports this sm version
 * (e.g. 90) in the capability checks; 0 restores the real query.
 * svdq_test_bounded_wait: launch a one-CTA kernel that waits, with the same
 * bounded-wait routine the kernels use, on an mbarrier nothing arrives on, for
 * at most timeout_ns; writes the kernel's status word (nonzero = gave up) to
 * *status_out and synchronizes the stream.  Faults, traps or hangs nothing.
 */
SVDQ_API void svdq_test_override_device_arch(int sm);
SVDQ_API svdq_status svdq_test_bounded_wait(uint64_t timeout_ns, uint32_t* status_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H */
