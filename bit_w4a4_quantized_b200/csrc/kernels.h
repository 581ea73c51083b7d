// kernels.h -- host-side launch interface of the CUDA kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/svdq.h"
#include "layout.h"

namespace svdq {

// Kernel 1: smoothing + NVFP4 quantization of X + down projection.
struct ActQuantLaunch {
  const void* X;         // device bf16 [M, K]
  const uint8_t* layer;  // device layer image
  uint8_t* act;          // device activation buffer
  LayerGeom lg;
  int64_t M;
  int32_t r_tot;         // ranks in use (0: no low-rank branch)
  float g_a, c_a, inv_alpha;
  int num_sms;
  uint64_t timeout_ns;
  int32_t int4;          // INT4 layer: groups of 64 with bf16 scales (int4.h) instead of NVFP4
};
cudaError_t launch_act_quant(const ActQuantLaunch& a, cudaStream_t s, const char** why);

// Kernel 2: block-scaled NVFP4 GEMM + low-rank up projection + epilogue.
struct GemmLaunch {
  const uint8_t* act;    // device activation buffer (filled by kernel 1)
  const uint8_t* layer;  // device layer image
  void* Y;               // device bf16 [M, N]
  LayerGeom lg;
  int64_t M;
  int32_t r_tot;
  int32_t has_bias;
  int32_t epilogue;
  float alpha;
  int num_sms;
  uint64_t timeout_ns;
  // fused QKV epilogue (qkv_cols = N / 3 > 0): per-head RMSNorm of Q and K,
  // rotary turn of their pairs; V unchanged.  head_dim 128.
  int32_t qkv_cols;
  const uint16_t* norm_q;  // device bf16 [128]
  const uint16_t* norm_k;  // device bf16 [128]
  const float* rope;       // device packed rotary table (rope_packed_bytes(M) bytes)
  float eps;
  // fused MLP pair (mlp_act2 != null): instead of Y, the epilogue writes the next layer's
  // (fc2's) NVFP4 codes and block scales of x_hat2 = bf16(y bf16 / lambda2) into its
  // activation buffer, and per weight tile the partial x_hat2 L1_2 into mlp_partial
  // [NT][MT * 128][r2] (fp32); launch_mlp_reduce then sums the partials into fc2's lr'.
  uint8_t* mlp_act2;        // fc2's activation buffer
  const uint8_t* mlp_layer2; // fc2's device image
  LayerGeom mlp_lg2;
  int32_t mlp_r2;           // fc2's ranks in use
  float mlp_g_a2, mlp_c_a2;
  float* mlp_partial;
};
cudaError_t launch_gemm(const GemmLaunch& a, cudaStream_t s, const char** why);

// Fused MLP pair, second step: lr'2[m][rho] = bf16(sum over weight tiles t of
// partial[t][m][rho] / alpha2) into fc2's activation buffer, tiles in a fixed order.
struct MlpReduceLaunch {
  const float* partial;  // [nt][rows][r2]
  int32_t nt;            // weight tiles of fc1 (partials per row)
  int64_t rows;          // MT * 128 rows of fc2's activation buffer
  int32_t r2;
  float inv_alpha2;
  uint8_t* lr2;          // fc2's act buffer + off_lr
  int32_t RJ2;           // fc2's low-rank chunks per row tile
};
cudaError_t launch_mlp_reduce(const MlpReduceLaunch& a, cudaStream_t s);

// The library's static scratch for the fused MLP pair of callers that cannot allocate
// (mlp_static.cu): its device address on device `dev`, looked up once per device with that
// device current.
constexpr size_t kMlpStaticBytes = size_t(SVDQ_MLP_STATIC_SCRATCH_BYTES);
cudaError_t mlp_static_scratch(int dev, void** ptr);
size_t mlp_partial_bytes(int64_t NT1, int64_t MT, int32_t r2);

// [M][64][2] float (cos, sin) -> the packed layout of rope_packed_bytes(M).
cudaError_t launch_rope_pack(const float* rope, int64_t M, float* packed, cudaStream_t s);

// LoRA attach/detach: rewrite ranks [rank, rank_capacity) of L1^T and L2^T.
struct LoraLaunch {
  uint8_t* layer;
  LayerGeom lg;
  const uint16_t* A;  // device bf16 [K, r_e] or NULL when r_e == 0
  const uint16_t* B;  // device bf16 [r_e, N]
  int32_t r_e;
  float scale;
};
cudaError_t launch_lora_swap(const LoraLaunch& a, cudaStream_t s);

// Test hook: bounded wait on an mbarrier nothing arrives on.
cudaError_t run_bounded_wait_test(uint64_t timeout_ns, uint32_t* status_out, cudaStream_t s);

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait

}  // namespace svdq
