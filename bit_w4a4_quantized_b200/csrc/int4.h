// int4.h -- the INT4 variant of the 4-bit layer (the Diffusers/Nunchaku page's
// svdq_w4a4 family comes in INT4 and NVFP4 variants; --precision int4 picks
// this one): byte layouts of its codes and scales, and its kernels' launches.
//
// Format: one bf16 scale per group of 64 consecutive elements along K, codes
// q = -7 .. 7 (q_max = 7 in the summary page's quantizer round(X / s),
// s = max|X| / q_max) as two's-complement nibbles, element 2i of a byte pair
// in the low nibble.
//
// The INT4 layer reuses the NVFP4 layer's geometry (LayerGeom, ActGeom): its
// codes take the same 4 bits per element, and its scales (2 bytes per 64
// elements) half of the NVFP4 scale region.  Inside those regions:
//   * codes: blocks of 128 rows x one group of 64, 4 KB each, laid out as
//     [2 halves of the group][128 rows][16 bytes], so that the 16-byte reads of
//     128 consecutive rows touch every shared-memory bank once;
//       weights:     [N / 256][KC][2 row halves of the 256-row tile][block]
//       activations: [M / 128 (padded)][KC][block]
//   * scales: bf16 [tile][KC][rows of the tile] (256 weight rows, 128 activation rows).
// Groups past K (KC counts 64-element chunks up to K rounded to 256) hold zeros.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.h"

namespace svdq {

constexpr int kGroup4 = 64;                        // elements per INT4 scale
constexpr uint32_t kBlock4Bytes = 128 * 32;        // 128 rows x 64 codes
constexpr uint32_t kScale4Bytes = 128 * 2;         // 128 rows x one bf16 scale

// byte holding elements (k, k + 1) (k even) of row i (0..127) inside a 4 KB block
SVDQ_HD uint32_t int4_block_byte(uint32_t i, uint32_t k) { return ((k % 64) / 32) * 2048u + i * 16u + (k % 32) / 2; }

SVDQ_HD size_t int4_bcode_off(const LayerGeom& g, int64_t n, int64_t k) {
  const size_t blk = (size_t(n / kBN) * size_t(g.KC) + size_t(k / kGroup4)) * 2 + size_t((n % kBN) / 128);
  return g.off_bcodes + blk * kBlock4Bytes + int4_block_byte(uint32_t(n % 128), uint32_t(k));
}
SVDQ_HD size_t int4_bsf_off(const LayerGeom& g, int64_t n, int64_t c) {
  return g.off_sfb + ((size_t(n / kBN) * size_t(g.KC) + size_t(c)) * kBN + size_t(n % kBN)) * 2;
}
SVDQ_HD size_t int4_acode_off(const ActGeom& a, int64_t m, int64_t k) {
  const size_t blk = size_t(m / kBM) * size_t(a.KT * 4) + size_t(k / kGroup4);
  return a.off_codes + blk * kBlock4Bytes + int4_block_byte(uint32_t(m % kBM), uint32_t(k));
}
SVDQ_HD size_t int4_asf_off(const ActGeom& a, int64_t m, int64_t c) {
  return a.off_sf + ((size_t(m / kBM) * size_t(a.KT * 4) + size_t(c)) * kBM + size_t(m % kBM)) * 2;
}

// Kernel 2 of the INT4 layer: the tensor cores take f16 operands, so each
// stage's codes are widened in shared memory to q * s * 2^e (exact in f16 for a
// bf16 scale s within f16's normal range), with a power-of-two prescale per
// operand (e_a for the activations, from the calibration maximum; e_w for the
// weights, from their largest scale) that keeps the values inside f16's range;
// alpha = 2^-(e_a + e_w) takes it back out in the epilogue.
struct Int4GemmLaunch {
  const uint8_t* act;    // device activation buffer (filled by kernel 1's INT4 instance)
  const uint8_t* layer;  // device layer image
  void* Y;               // device bf16 [M, N]
  LayerGeom lg;
  int64_t M;
  int32_t r_tot;
  int32_t has_bias;
  int32_t epilogue;
  float alpha;           // 2^-(e_a + e_w)
  float pre_a, pre_w;    // 2^e_a, 2^e_w
  int num_sms;
  uint64_t timeout_ns;
};
cudaError_t launch_gemm_int4(const Int4GemmLaunch& a, cudaStream_t s, const char** why);

}  // namespace svdq
