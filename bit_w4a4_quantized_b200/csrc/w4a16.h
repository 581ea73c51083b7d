// w4a16.h -- the W4A16 layer (4-bit NVFP4 weights, bf16 activations): the
// awq_w4a16 kernel family of the Diffusers/Nunchaku page, used there for the
// memory-bound adaptive-norm and modulation projections.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <string>
#include <vector>

#include "svdq.h"

namespace svdq {

// Device image of one W4A16 layer (one caller buffer, 256-byte aligned sections):
//   status word | 1/s float [K] | bias bf16 [N] | codes [N][K/2] | scales [N][K/16]
// Codes: E2M1, element 2i in the low nibble of byte i of its row.  Scales: E4M3.
struct W4A16Geom {
  int64_t K, N;
  size_t off_inv_s, off_bias, off_codes, off_scales, total;
};
W4A16Geom make_w4a16_geom(int64_t K, int64_t N);

struct W4A16Launch {
  const uint8_t* layer;  // device image
  W4A16Geom g;
  const uint16_t* X;  // device bf16 [M, K]
  int64_t M;
  uint16_t* Y;  // device bf16 [M, N]
  float gscale;
  int32_t has_bias;
  int num_sms;
};
cudaError_t launch_w4a16(const W4A16Launch& a, cudaStream_t s, const char** why);

// Host quantization: fills `image` (host copy of the device image) and *g.
svdq_status w4a16_quantize(const svdq_w4a16_desc* d, std::vector<uint8_t>* image, float* g, std::string* err);

}  // namespace svdq

struct svdq_w4a16 {
  svdq::W4A16Geom g;
  std::vector<uint8_t> image;  // host copy of the device image
  float gscale = 1.0f;
  bool has_bias = false;
  void* dev_buf = nullptr;
  int device = -1;
  int num_sms = 0;
};
