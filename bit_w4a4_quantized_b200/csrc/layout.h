// layout.h -- tile geometry and byte layouts shared by the host packer and the kernels.
//
// Every operand of the tensor-core MMAs is stored in global memory already in
// the exact shared-memory image the MMA reads (K-major rows of 128 bytes, the
// 128-byte swizzle, 8-row atoms of 1 KB), one contiguous block per tile.  A
// pipeline stage is then filled by a handful of 1D bulk copies
// (cp.async.bulk), with no tensor map, no 2D addressing and no alignment
// corner cases.  The one operand that arrives in the caller's layout (X, row
// major) is read with a 2D TMA tensor load that applies the same swizzle.
//
// Block scales use the 128-row x 4-scale atom of 512 bytes the block-scaled
// MMA consumes from tensor memory: scale g (0..3) of row i (0..127) of a
// 64-element K block sits at byte (i % 32) * 16 + (i / 32) * 4 + g.
#pragma once

#include <stddef.h>
#include <stdint.h>

#if defined(__CUDACC__)
#define SVDQ_HD __host__ __device__ __forceinline__
#else
#define SVDQ_HD inline
#endif

namespace svdq {

constexpr int kBM = 128;           // activation rows per tile (MMA M)
constexpr int kBN = 256;           // weight rows (output features) per tile (MMA N)
constexpr int kBK = 256;           // K elements per GEMM k-tile: 128 bytes of E2M1 per row
constexpr int kKChunk = 64;        // K elements per quantizer chunk: 128 bytes of bf16 per row
constexpr int kRChunk = 64;        // ranks per low-rank chunk: 128 bytes of bf16 per row
constexpr int kRowBytes = 128;     // every tiled operand row is 128 bytes
constexpr int kATileBytes = kBM * kRowBytes;          // 16 KB
constexpr int kBTileBytes = kBN * kRowBytes;          // 32 KB
constexpr int kSFAtomBytes = 512;                     // 128 rows x 4 scales
constexpr int kSFATileBytes = 4 * kSFAtomBytes;       // 128 rows x 16 scales (one k-tile)
constexpr int kSFBTileBytes = 8 * kSFAtomBytes;       // 256 rows x 16 scales
constexpr int kMaxRankCapacity = 256;
constexpr int kStatusBytes = 256;

SVDQ_HD int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
SVDQ_HD int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
SVDQ_HD size_t align256(size_t a) { return (a + 255) & ~size_t(255); }

// Rotary table of the fused QKV epilogue (head_dim 128), packed so that the
// epilogue's lanes (one output row each) read consecutive 16 bytes:
//   [row tile t (an even count, like the GEMM's)][chunk c][row i of the tile]
// of 16 bytes = (cos, sin) of pairs 2c and 2c + 1 of row 128 t + i (zeros
// past the last row).
constexpr int kRopeHeadDim = 128;
constexpr int kRopeChunks = kRopeHeadDim / 4;  // 32 chunks of 2 pairs
SVDQ_HD size_t rope_packed_bytes(int64_t M) {
  return size_t(round_up(ceil_div(M, kBM), 2)) * kRopeChunks * kBM * 16;
}

// Byte offset, inside a tile of 128-byte rows, of byte `b` (0..127) of row
// `row` under the 128-byte swizzle: the 16-byte chunk index is XORed with row % 8.
SVDQ_HD uint32_t sw128(uint32_t row, uint32_t b) {
  return row * 128u + ((((b >> 4) ^ (row & 7u)) << 4) | (b & 15u));
}

// Byte offset inside a 512-byte scale atom of scale g (0..3) of row i (0..127).
SVDQ_HD uint32_t sf_atom(uint32_t i, uint32_t g) { return (i & 31u) * 16u + (i >> 5) * 4u + g; }

// ---------------------------------------------------------------- layer image
struct LayerGeom {
  int64_t K, N;
  int32_t rank, rcap;   // base rank and rank capacity (multiples of 16)
  int64_t KT;           // k-tiles of 256
  int64_t KC;           // quantizer chunks of 64 = 4 * KT
  int64_t NT;           // weight tiles of 256 rows
  int64_t RC16;         // rows of one L1^T chunk = rcap
  int64_t RJ;           // low-rank chunks of 64 ranks = ceil(rcap / 64)
  size_t off_status, off_lam, off_inv_lam, off_bias, off_bcodes, off_sfb, off_l1t, off_l2t;
  size_t total;
};

SVDQ_HD LayerGeom make_layer_geom(int64_t K, int64_t N, int32_t rank, int32_t rcap) {
  LayerGeom g{};
  g.K = K;
  g.N = N;
  g.rank = rank;
  g.rcap = rcap;
  g.KT = ceil_div(K, kBK);
  g.KC = g.KT * (kBK / kKChunk);
  g.NT = ceil_div(N, kBN);
  g.RC16 = rcap;
  g.RJ = ceil_div(rcap, kRChunk);
  size_t o = 0;
  g.off_status = o;  o += kStatusBytes;
  g.off_lam = o;     o = align256(o + size_t(g.KC) * kKChunk * 4);
  g.off_inv_lam = o; o = align256(o + size_t(g.KC) * kKChunk * 4);
  g.off_bias = o;    o = align256(o + size_t(g.NT) * kBN * 2);
  g.off_bcodes = o;  o = align256(o + size_t(g.NT) * g.KT * kBTileBytes);
  g.off_sfb = o;     o = align256(o + size_t(g.NT) * g.KT * kSFBTileBytes);
  g.off_l1t = o;     o = align256(o + size_t(g.KC) * g.RC16 * kRowBytes);
  g.off_l2t = o;     o = align256(o + size_t(g.NT) * g.RJ * kBTileBytes);
  g.total = o;
  return g;
}

// weight codes: byte holding elements (k, k+1) (k even) of output row n
SVDQ_HD size_t bcode_off(const LayerGeom& g, int64_t n, int64_t k) {
  size_t tile = size_t(n / kBN) * g.KT + size_t(k / kBK);
  return g.off_bcodes + tile * kBTileBytes + sw128(uint32_t(n % kBN), uint32_t((k % kBK) / 2));
}
// weight block scale of output row n, K block s (= k / 16)
SVDQ_HD size_t bsf_off(const LayerGeom& g, int64_t n, int64_t s) {
  size_t tile = size_t(n / kBN) * g.KT + size_t(s / 16);
  uint32_t kb = uint32_t((s % 16) / 4), h = uint32_t((n % kBN) / 128);
  return g.off_sfb + tile * kSFBTileBytes + (kb * 2 + h) * kSFAtomBytes +
         sf_atom(uint32_t(n % 128), uint32_t(s % 4));
}
// L1^T (rank rho, input feature k), bf16
SVDQ_HD size_t l1t_off(const LayerGeom& g, int64_t rho, int64_t k) {
  return g.off_l1t + size_t(k / kKChunk) * size_t(g.RC16) * kRowBytes +
         sw128(uint32_t(rho), uint32_t((k % kKChunk) * 2));
}
// L2^T (output feature n, rank rho), bf16
SVDQ_HD size_t l2t_off(const LayerGeom& g, int64_t n, int64_t rho) {
  size_t tile = size_t(n / kBN) * g.RJ + size_t(rho / kRChunk);
  return g.off_l2t + tile * kBTileBytes + sw128(uint32_t(n % kBN), uint32_t((rho % kRChunk) * 2));
}

// ---------------------------------------------------------- activation buffer
// Rows are padded to an even number of 128-row tiles; the padding rows hold
// zero codes and scales (kernel 1 reads them as zeros past the end of X).
struct ActGeom {
  int64_t M, MT, KT, RJ;
  size_t off_codes, off_sf, off_lr, total;
};

SVDQ_HD ActGeom make_act_geom(const LayerGeom& lg, int64_t M) {
  ActGeom a{};
  a.M = M;
  a.MT = round_up(ceil_div(M, kBM), 2);  // the GEMM works on pairs of 128-row tiles
  a.KT = lg.KT;
  a.RJ = lg.RJ;
  size_t o = 0;
  a.off_codes = o; o = align256(o + size_t(a.MT) * a.KT * kATileBytes);
  a.off_sf = o;    o = align256(o + size_t(a.MT) * a.KT * kSFATileBytes);
  a.off_lr = o;    o = align256(o + size_t(a.MT) * a.RJ * kATileBytes);
  a.total = o;
  return a;
}

SVDQ_HD size_t acode_off(const ActGeom& a, int64_t m, int64_t k) {
  size_t tile = size_t(m / kBM) * a.KT + size_t(k / kBK);
  return a.off_codes + tile * kATileBytes + sw128(uint32_t(m % kBM), uint32_t((k % kBK) / 2));
}
SVDQ_HD size_t asf_off(const ActGeom& a, int64_t m, int64_t s) {
  size_t tile = size_t(m / kBM) * a.KT + size_t(s / 16);
  return a.off_sf + tile * kSFATileBytes + uint32_t((s % 16) / 4) * kSFAtomBytes +
         sf_atom(uint32_t(m % kBM), uint32_t(s % 4));
}
SVDQ_HD size_t lr_off(const ActGeom& a, int64_t m, int64_t rho) {
  size_t tile = size_t(m / kBM) * a.RJ + size_t(rho / kRChunk);
  return a.off_lr + tile * kATileBytes + sw128(uint32_t(m % kBM), uint32_t((rho % kRChunk) * 2));
}

}  // namespace svdq
