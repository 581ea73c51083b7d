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
//   status word | 1/s float [K] | bias bf16 [N] | codes | scales
// The weights are cut into tiles of 16 rows x 64 inputs, stored tile after tile
// (row tile major), each in the order the tensor-core fragments want them:
//   codes: 512 bytes per tile = 32 lanes x 16 bytes; lane t = 4 g + c holds,
//     for the tile's four 16-input steps j, the 4 bytes (rows g, g + 8 at
//     inputs 16 j + 2 c, then rows g, g + 8 at 16 j + 2 c + 8), two E2M1
//     codes per byte, the lower input in the low nibble;
//   scales: 64 bytes per tile = 8 groups g x 8 bytes: the E4M3 scales of rows
//     g (steps 0..3), then g + 8 (steps 0..3).
// Rows past N are zero.
struct W4A16Geom {
  int64_t K, N, N16, KT;  // N16 = N rounded up to 16; KT = K / 64
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
  uint64_t timeout_ns;  // per bounded wait; a timeout sets the image's status word
};
cudaError_t launch_w4a16(const W4A16Launch& a, cudaStream_t s, const char** why);

// Host quantization: fills `image` (host copy of the device image), the
// row-major codes [N][K/2] and scales [N][K/16] (for exports) and *g.
svdq_status w4a16_quantize(const svdq_w4a16_desc* d, std::vector<uint8_t>* image, std::vector<uint8_t>* codes,
                           std::vector<uint8_t>* scales, float* g, std::string* err);

}  // namespace svdq

struct svdq_w4a16 {
  svdq::W4A16Geom g;
  std::vector<uint8_t> image;  // host copy of the device image
  std::vector<uint8_t> codes;  // row-major [N][K/2], for exports
  std::vector<uint8_t> scales;  // row-major [N][K/16], for exports
  float gscale = 1.0f;
  bool has_bias = false;
  void* dev_buf = nullptr;
  int device = -1;
  int num_sms = 0;
};
