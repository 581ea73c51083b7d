// w4a16.cu -- the W4A16 layer's kernel: Y = g x~ deq(W')^T + b with 4-bit NVFP4
// weights W' = W diag(s) and x~ = f16(x / s), for the small batches of the
// modulation projections (Diffusers/Nunchaku page: awq_w4a16, memory bound).
//
// Design (sm_100a): the kernel streams the 4-bit weights once, so its roofline
// is HBM bandwidth; the arithmetic only has to stay out of the way.  It runs on
// the tensor cores with the warp-level m16n8k16 MMA (f16 operands, float32
// accumulators): A = 16 weight rows x 16 inputs, dequantized in registers (the
// hardware E2M1 -> f16x2 conversion, times the E4M3 block scale: exact in f16),
// B = 16 inputs x 8 rows of X (x~ in shared memory; rows past M are zero
// operands in registers).  The prepared image stores each 16 x 64 weight tile
// in fragment order, so one 16-byte load per lane brings the A operands of
// four MMAs.  A CTA of 8 warps takes a 16-row tile of the output; its warps
// split K (tile kt goes to warp kt % 8), issue all their weight loads before
// any arithmetic, and add their partial sums through shared memory in a fixed
// order.  With one row of X the MMA would be 7/8 padding, so that launch does
// the same tiles on the CUDA cores instead: mixed-precision fused multiply-adds
// (f16 operands, float32 accumulator) straight from the f16 weights, no
// conversion to float32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>

#include "layout.h"
#include "w4a16.h"

namespace svdq {

W4A16Geom make_w4a16_geom(int64_t K, int64_t N) {
  W4A16Geom g{};
  g.K = K;
  g.N = N;
  g.N16 = (N + 15) / 16 * 16;
  g.KT = K / 64;
  size_t o = kStatusBytes;
  g.off_inv_s = o;
  o = align256(o + size_t(K) * 4);
  g.off_bias = o;
  o = align256(o + size_t(N) * 2);
  g.off_codes = o;
  o = align256(o + size_t(g.N16) * size_t(K / 2));
  g.off_scales = o;
  o = align256(o + size_t(g.N16) * size_t(K / 16));
  g.total = o;
  return g;
}

namespace {

constexpr int kThreadsW = 256;  // 8 warps
constexpr int kWarpsW = kThreadsW / 32;
constexpr int kMaxMW = 8;  // rows of X per launch: the MMA's N
constexpr int kTilesPerWarp = 6;  // weight tiles whose loads a warp issues together (K = 3072: all of them)

struct W4A16Params {
  const uint4* codes;   // [N16 / 16][KT][32 lanes] x 16 bytes
  const uint2* scales;  // [N16 / 16][KT][8 groups] x 8 bytes
  const float* inv_s;
  const uint16_t* bias;  // or null
  const uint16_t* X;
  uint16_t* Y;
  int64_t K, N, M, NT, KT;
  float g;
};

// Four code bytes (8 E2M1 codes, each byte's first in its low nibble) -> four
// f16x2, byte i in h[i], its first code in the low half.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t* h) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}
// Four E4M3 scales (one word) -> two f16x2: {s0, s1} and {s2, s3}.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n cvt.rn.f16x2.e4m3x2 %0, l;\n cvt.rn.f16x2.e4m3x2 %1, h;\n}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}
// The low (j = 0) or high (j = 1) half of an f16x2, in both halves.
__device__ __forceinline__ uint32_t dup_half(uint32_t v, int j) { return __byte_perm(v, 0u, j ? 0x3232u : 0x1010u); }
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// D = A B + D, m16n8k16, f16 operands, float32 accumulators.
__device__ __forceinline__ void mma_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 16 x 64 weight tile against x~: 4 MMAs.  cw: this lane's 16 code bytes;
// sw: the 8 scale bytes of its rows g (x) and g + 8 (y); xrow: x~ row g as
// f16 pairs, at the tile's first input, or null when row g of X is past M.
__device__ __forceinline__ void tile_mma(float* acc, uint4 cw, uint2 sw, const uint32_t* xrow, int c) {
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
  uint32_t sg[2], sg8[2];  // scales of rows g and g + 8: steps {0, 1}, {2, 3}
  e4m3x4_to_f16x2(sw.x, sg[0], sg[1]);
  e4m3x4_to_f16x2(sw.y, sg8[0], sg8[1]);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t h[4];
    e2m1x8_to_f16x2(words[j], h);
    const uint32_t s0 = dup_half(sg[j >> 1], j & 1);   // row g
    const uint32_t s1 = dup_half(sg8[j >> 1], j & 1);  // row g + 8
    const uint32_t a0 = hmul2(h[0], s0);
    const uint32_t a1 = hmul2(h[1], s1);
    const uint32_t a2 = hmul2(h[2], s0);
    const uint32_t a3 = hmul2(h[3], s1);
    const uint32_t b0 = xrow ? xrow[8 * j + c] : 0u;      // inputs 16 j + 2 c, + 1
    const uint32_t b1 = xrow ? xrow[8 * j + c + 4] : 0u;  // inputs 16 j + 2 c + 8, + 9
    mma_16816(acc, a0, a1, a2, a3, b0, b1);
  }
}

// acc + x.lo w.lo + x.hi w.hi with f16 operands and a float32 accumulator
// (exact products, float32 sums).
__device__ __forceinline__ float fma2_f16_f32(uint32_t x2, uint32_t w2, float acc) {
  asm("{\n .reg .f16 xl, xh, wl, wh;\n mov.b32 {xl, xh}, %1;\n mov.b32 {wl, wh}, %2;\n"
      " fma.rn.f32.f16 %0, xl, wl, %0;\n fma.rn.f32.f16 %0, xh, wh, %0;\n}"
      : "+f"(acc)
      : "r"(x2), "r"(w2));
  return acc;
}

// The same 16 x 64 tile on the CUDA cores, for kM <= 2 rows of X (the MMA's 8
// columns would be mostly padding): lane (g, c) adds its 16 weights of rows g
// (acc[0][m]) and g + 8 (acc[1][m]) times x~; xs: x~ rows as f16 pairs, at the
// tile's first input.
template <int kM>
__device__ __forceinline__ void tile_dot(float (*acc)[kM], uint4 cw, uint2 sw, const uint32_t* xs, uint32_t RW,
                                         int c) {
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
  uint32_t sg[2], sg8[2];  // scales of rows g and g + 8: steps {0, 1}, {2, 3}
  e4m3x4_to_f16x2(sw.x, sg[0], sg[1]);
  e4m3x4_to_f16x2(sw.y, sg8[0], sg8[1]);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t h[4];
    e2m1x8_to_f16x2(words[j], h);
    const uint32_t s0 = dup_half(sg[j >> 1], j & 1);   // row g
    const uint32_t s1 = dup_half(sg8[j >> 1], j & 1);  // row g + 8
    const uint32_t a0 = hmul2(h[0], s0);  // row g, inputs 16 j + 2 c, + 1
    const uint32_t a1 = hmul2(h[1], s1);  // row g + 8, the same inputs
    const uint32_t a2 = hmul2(h[2], s0);  // row g, inputs 16 j + 2 c + 8, + 9
    const uint32_t a3 = hmul2(h[3], s1);  // row g + 8, the same inputs
#pragma unroll
    for (int m = 0; m < kM; ++m) {
      const uint32_t x0 = xs[m * RW + 8 * j + c], x1 = xs[m * RW + 8 * j + c + 4];
      acc[0][m] = fma2_f16_f32(x1, a2, fma2_f16_f32(x0, a0, acc[0][m]));
      acc[1][m] = fma2_f16_f32(x1, a3, fma2_f16_f32(x0, a1, acc[1][m]));
    }
  }
}

// kDot = 0: the MMA path (2 to 8 rows of X); kDot = 1: the CUDA-core path for one row.
// The one-row instance fits 64 registers, so 4 CTAs share an SM (measured 15.2 -> 14.6 us at K = 3072,
// N = 18432).  The MMA instance is faster with room for 106 registers and 2 CTAs per SM (M = 4:
// 18.7 -> 17.3 us) than held to 80 registers and 3.
template <int kDot>
__global__ void __launch_bounds__(kThreadsW, kDot ? 4 : 1) w4a16_kernel(const W4A16Params p) {
  extern __shared__ uint32_t smem_w[];
  const int64_t K = p.K;
  const uint32_t RW = uint32_t(K / 2) + 4;  // x~ row stride in f16 pairs (+4: rows start on different banks)
  const uint32_t MR = uint32_t(p.M);        // rows of x~ kept (B columns past M are zero in registers)
  uint32_t* xs = smem_w;                    // [M][RW] f16 pairs
  float* red = reinterpret_cast<float*>(smem_w + MR * RW);  // [8 warps][32 lanes][4]
  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const int g = lane >> 2, c = lane & 3;

  // the first tile's weight loads go out before x~ is staged
  int64_t nt = blockIdx.x;
  uint4 cw[kTilesPerWarp];
  uint2 sw[kTilesPerWarp];
  auto load = [&](int64_t tile, int64_t kt0) {
#pragma unroll
    for (int i = 0; i < kTilesPerWarp; ++i) {
      const int64_t kt = kt0 + int64_t(i) * kWarpsW;
      if (tile < p.NT && kt < p.KT) {
        cw[i] = __ldg(p.codes + (tile * p.KT + kt) * 32 + lane);
        sw[i] = __ldg(p.scales + (tile * p.KT + kt) * 8 + g);
      } else {
        cw[i] = make_uint4(0u, 0u, 0u, 0u);
        sw[i] = make_uint2(0u, 0u);
      }
    }
  };
  load(nt, warp);

  // x~ = f16(x / s), saturating
  for (uint32_t i = threadIdx.x; i < MR * uint32_t(K / 2); i += kThreadsW) {
    const uint32_t m = i / uint32_t(K / 2), w = i % uint32_t(K / 2);
    const uint32_t xb = *reinterpret_cast<const uint32_t*>(p.X + int64_t(m) * K + 2 * int64_t(w));
    const float2 is = *reinterpret_cast<const float2*>(p.inv_s + 2 * int64_t(w));
    const float lo = fminf(fmaxf(__uint_as_float(xb << 16) * is.x, -65504.0f), 65504.0f);
    const float hi = fminf(fmaxf(__uint_as_float(xb & 0xFFFF0000u) * is.y, -65504.0f), 65504.0f);
    const __half2 h = __floats2half2_rn(lo, hi);
    xs[m * RW + w] = *reinterpret_cast<const uint32_t*>(&h);
  }
  __syncthreads();

  for (; nt < p.NT; nt += gridDim.x) {
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float dacc[2][kDot > 0 ? kDot : 1] = {};
    const uint32_t* xrow = uint32_t(g) < MR ? xs + uint32_t(g) * RW : nullptr;
    for (int64_t kt0 = warp;; kt0 += int64_t(kTilesPerWarp) * kWarpsW) {
#pragma unroll
      for (int i = 0; i < kTilesPerWarp; ++i) {
        const int64_t kt = kt0 + int64_t(i) * kWarpsW;
        if (kt < p.KT) {
          if constexpr (kDot > 0)
            tile_dot<kDot>(dacc, cw[i], sw[i], xs + uint32_t(kt) * 32u, RW, c);
          else
            tile_mma(acc, cw[i], sw[i], xrow ? xrow + uint32_t(kt) * 32u : nullptr, c);
        }
      }
      const int64_t next = kt0 + int64_t(kTilesPerWarp) * kWarpsW;
      if (next < p.KT) {
        load(nt, next);  // more of this row tile (K > 3072)
      } else {
        load(nt + gridDim.x, warp);  // the next row tile's first loads overlap the reduction
        break;
      }
    }
    if constexpr (kDot > 0) {
      // the 4 lanes of a row group hold disjoint inputs: add them (lane c = 0 keeps the sums), then lay
      // the result out as the MMA accumulator would hold it: lane (g, c) row g (x, y), row g + 8 (z, w),
      // X rows 2 c, 2 c + 1
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < kDot; ++m) {
          dacc[h][m] += __shfl_xor_sync(0xFFFFFFFFu, dacc[h][m], 1);
          dacc[h][m] += __shfl_xor_sync(0xFFFFFFFFu, dacc[h][m], 2);
        }
      acc[0] = c == 0 ? dacc[0][0] : 0.0f;
      acc[2] = c == 0 ? dacc[1][0] : 0.0f;
      acc[1] = (c == 0 && kDot > 1) ? dacc[0][kDot > 1 ? 1 : 0] : 0.0f;
      acc[3] = (c == 0 && kDot > 1) ? dacc[1][kDot > 1 ? 1 : 0] : 0.0f;
    }
    // the 8 warps' partial tiles, added in warp order
    *reinterpret_cast<float4*>(red + (warp * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (warp == 0) {
      float4 t = *reinterpret_cast<const float4*>(red + lane * 4);
#pragma unroll
      for (int w = 1; w < kWarpsW; ++w) {
        const float4 u = *reinterpret_cast<const float4*>(red + (w * 32 + lane) * 4);
        t.x += u.x;
        t.y += u.y;
        t.z += u.z;
        t.w += u.w;
      }
      // lane (g, c): rows n = 16 nt + g (x, y) and + 8 (z, w); X rows m = 2 c (x, z) and 2 c + 1 (y, w)
      const float v[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t n = nt * 16 + g + 8 * (q >> 1);
        const int64_t m = 2 * c + (q & 1);
        if (n < p.N && m < p.M) {
          const float b = p.bias ? __uint_as_float(uint32_t(p.bias[n]) << 16) : 0.0f;
          const __nv_bfloat16 y = __float2bfloat16_rn(fmaf(p.g, v[q], b));
          p.Y[m * p.N + n] = *reinterpret_cast<const uint16_t*>(&y);
        }
      }
    }
    __syncthreads();  // red is rewritten by the next row tile
  }
}

// Blocks per SM for this device and shared-memory size, queried once (the
// attribute and occupancy calls cost microseconds of host time; a launch
// should not).  The carveout asks for all of the unified L1 as shared memory,
// or the driver may size it for one CTA.
template <int kDot>
int blocks_per_sm(size_t smem) {
  static std::atomic<int64_t> cached_key[64];
  static std::atomic<int> cached_val[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int64_t key = int64_t(smem) + 1;
  if (cached_key[dev & 63].load() == key) return cached_val[dev & 63].load();
  if (cudaFuncSetAttribute(w4a16_kernel<kDot>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess ||
      cudaFuncSetAttribute(w4a16_kernel<kDot>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           int(cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
    return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, w4a16_kernel<kDot>, kThreadsW, smem) != cudaSuccess)
    return 0;
  cached_val[dev & 63].store(per_sm);
  cached_key[dev & 63].store(key);
  return per_sm;
}

}  // namespace

cudaError_t launch_w4a16(const W4A16Launch& a, cudaStream_t s, const char** why) {
  W4A16Params p{};
  p.codes = reinterpret_cast<const uint4*>(a.layer + a.g.off_codes);
  p.scales = reinterpret_cast<const uint2*>(a.layer + a.g.off_scales);
  p.inv_s = reinterpret_cast<const float*>(a.layer + a.g.off_inv_s);
  p.bias = a.has_bias ? reinterpret_cast<const uint16_t*>(a.layer + a.g.off_bias) : nullptr;
  p.K = a.g.K;
  p.N = a.g.N;
  p.NT = a.g.N16 / 16;
  p.KT = a.g.KT;
  p.g = a.gscale;
  // rows of X in launches of at most 8 (the MMA's N), stream ordered
  for (int64_t m0 = 0; m0 < a.M; m0 += kMaxMW) {
    p.X = a.X + m0 * a.g.K;
    p.Y = a.Y + m0 * a.g.N;
    p.M = a.M - m0 < kMaxMW ? a.M - m0 : kMaxMW;
    const size_t smem = (size_t(p.M) * size_t(a.g.K / 2 + 4) + size_t(kThreadsW) * 4) * 4;
    const int per_sm = p.M == 1 ? blocks_per_sm<1>(smem) : blocks_per_sm<0>(smem);
    if (per_sm < 1) {
      *why = "the W4A16 kernel does not fit on this device";
      return cudaErrorInvalidConfiguration;
    }
    int64_t blocks = int64_t(per_sm) * a.num_sms;
    if (blocks > p.NT) blocks = p.NT;
    if (p.M == 1)  // one row of X: the CUDA cores (measured 15 us against 18 us for the MMA at M = 1..4)
      w4a16_kernel<1><<<unsigned(blocks), kThreadsW, smem, s>>>(p);
    else
      w4a16_kernel<0><<<unsigned(blocks), kThreadsW, smem, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      *why = "launch of the W4A16 kernel failed";
      return e;
    }
  }
  return cudaSuccess;
}

}  // namespace svdq
