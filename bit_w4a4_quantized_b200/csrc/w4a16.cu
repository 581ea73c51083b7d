// w4a16.cu -- the W4A16 layer's kernel: Y = g (X diag(s)^-1) deq(W')^T + b with
// 4-bit NVFP4 weights and bf16 activations, for the small batches of the
// modulation projections (Diffusers/Nunchaku page: awq_w4a16, memory bound).
//
// Design (sm_100a): the kernel streams the weights once, so its roofline is
// HBM bandwidth.  A warp streams 4 weight rows at a time (2 when X has 3 or 4
// rows) and issues all of their loads for a 1024-weight step before any
// arithmetic: per step a lane reads 16 bytes of codes (32 weights) and their 2
// block scales of each row, so a warp reads 512 contiguous bytes per row.
// Every CTA keeps x~ = f32(x / s) for its rows of X in shared memory (16-byte
// chunks swizzled so the lanes' reads hit distinct banks); each x~ value a lane
// reads serves all the rows in flight, which keeps shared-memory traffic below
// the weight stream.  The E2M1 codes and
// E4M3 scales are decoded with the hardware f16x2 conversions (exact: every
// code times scale is an f16 value); the sums are float32, even and odd
// weights apart, one partial per 16-weight block, multiplied by the block
// scale.
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
  size_t o = kStatusBytes;
  g.off_inv_s = o;
  o = align256(o + size_t(K) * 4);
  g.off_bias = o;
  o = align256(o + size_t(N) * 2);
  g.off_codes = o;
  o = align256(o + size_t(N) * size_t(K / 2));
  g.off_scales = o;
  o = align256(o + size_t(N) * size_t(K / 16));
  g.total = o;
  return g;
}

namespace {

constexpr int kThreadsW = 256;  // 8 warps (128 measured slower)
constexpr int kMaxMW = 4;       // rows of X per launch

struct W4A16Params {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* inv_s;
  const uint16_t* bias;  // or null
  const uint16_t* X;
  uint16_t* Y;
  int64_t K, N, M;
  float g;
};

// Physical 16-byte chunk of logical chunk c of an x~ row: the 3 low bits are
// XORed with bits 3..5, so the 8 lanes of a quarter-warp, whose chunks are 8
// apart, read 8 different bank groups.
__device__ __forceinline__ uint32_t xswz(uint32_t c) { return c ^ ((c >> 3) & 7u); }

__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t& h0, uint32_t& h1, uint32_t& h2, uint32_t& h3) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
}
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t s) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(s));
  return h;
}
__device__ __forceinline__ float2 f16x2_to_f32(uint32_t h) {
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}
// The even and odd weights of a pair accumulate separately: (a.x b.x + c.x, a.y b.y + c.y).
// (The packed f32x2 fused multiply-add measured the same time as two scalar ones.)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
}

// Weight rows a warp streams at once: every x~ value read from shared memory
// serves all of them, so the shared-memory traffic per weight is 4 kM / kR bytes.
template <int kM>
__host__ __device__ constexpr int rows_in_flight() {
  return kM <= 2 ? 4 : 2;
}

// 1024-weight steps per lane whose loads are issued together.  More (3 cover
// K = 3072) was measured slower: the registers cost more occupancy than the
// extra loads in flight bought.
constexpr int kJ = 1;

// One 32-weight step of every row in flight: x~[m][c0 * 4 .. + 31] against
// the 16 code bytes cw[r] and 2 block scales sw[r] of row r; each x~ chunk read
// from shared memory serves all kR rows.
template <int kM, int kR>
__device__ __forceinline__ void step32(const float4* xs4, uint32_t KC, uint32_t c0, const uint4* cw,
                                       const uint16_t* sw, float2 (*acc)[kM]) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {  // two 16-weight blocks
    float2 part[kR][kM];
#pragma unroll
    for (int r = 0; r < kR; ++r)
#pragma unroll
      for (int m = 0; m < kM; ++m) part[r][m] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int wi = 0; wi < 2; ++wi) {  // 8 weights per code word
      const uint32_t c = c0 + uint32_t(4 * half + 2 * wi);
      float4 xa[kM], xb[kM];
#pragma unroll
      for (int m = 0; m < kM; ++m) {
        xa[m] = xs4[m * KC + xswz(c)];
        xb[m] = xs4[m * KC + xswz(c + 1)];
      }
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        const uint32_t word = half ? (wi ? cw[r].w : cw[r].z) : (wi ? cw[r].y : cw[r].x);
        uint32_t h[4];
        e2m1x8_to_f16x2(word, h[0], h[1], h[2], h[3]);
        const float2 w0 = f16x2_to_f32(h[0]), w1 = f16x2_to_f32(h[1]);
        const float2 w2 = f16x2_to_f32(h[2]), w3 = f16x2_to_f32(h[3]);
#pragma unroll
        for (int m = 0; m < kM; ++m) {
          part[r][m] = ffma2(make_float2(xa[m].x, xa[m].y), w0, part[r][m]);
          part[r][m] = ffma2(make_float2(xa[m].z, xa[m].w), w1, part[r][m]);
          part[r][m] = ffma2(make_float2(xb[m].x, xb[m].y), w2, part[r][m]);
          part[r][m] = ffma2(make_float2(xb[m].z, xb[m].w), w3, part[r][m]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kR; ++r) {
      const float2 sc = f16x2_to_f32(e4m3x2_to_f16x2(sw[r]));
      const float sv = half ? sc.y : sc.x;
#pragma unroll
      for (int m = 0; m < kM; ++m) acc[r][m] = ffma2(part[r][m], make_float2(sv, sv), acc[r][m]);
    }
  }
}

template <int kM>
__global__ void __launch_bounds__(kThreadsW) w4a16_kernel(const W4A16Params p) {
  constexpr int kR = rows_in_flight<kM>();
  extern __shared__ float4 xs4[];  // [kM][K / 4] chunks of x~, swizzled
  const int64_t K = p.K;
  const uint32_t KC = uint32_t(K / 4);
  // x~ = f32(x * (1 / s)) for this launch's rows
  for (uint32_t i = threadIdx.x; i < uint32_t(kM) * KC; i += kThreadsW) {
    const uint32_t m = i / KC, c = i % KC;
    const uint2 xb = *reinterpret_cast<const uint2*>(p.X + int64_t(m) * K + int64_t(c) * 4);
    const float4 is = *reinterpret_cast<const float4*>(p.inv_s + int64_t(c) * 4);
    float4 v;
    v.x = __uint_as_float(xb.x << 16) * is.x;
    v.y = __uint_as_float(xb.x & 0xFFFF0000u) * is.y;
    v.z = __uint_as_float(xb.y << 16) * is.z;
    v.w = __uint_as_float(xb.y & 0xFFFF0000u) * is.w;
    xs4[m * KC + xswz(c)] = v;
  }
  __syncthreads();

  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const int64_t nwarps = int64_t(gridDim.x) * (kThreadsW / 32);
  const int64_t row_bytes = K / 2, srow_bytes = K / 16;
  for (int64_t n0 = int64_t(blockIdx.x) * (kThreadsW / 32) + warp; n0 < p.N; n0 += kR * nwarps) {
    float2 acc[kR][kM];
#pragma unroll
    for (int r = 0; r < kR; ++r)
#pragma unroll
      for (int m = 0; m < kM; ++m) acc[r][m] = make_float2(0.0f, 0.0f);
    // lane l covers weights l * 32 .. + 31 of every 1024 along K; the loads of
    // kJ such steps for all kR rows are in flight before the arithmetic
    for (int64_t kb = 0; kb < K; kb += kJ * 1024) {
      uint4 cw[kJ][kR];
      uint16_t sw[kJ][kR];
#pragma unroll
      for (int j = 0; j < kJ; ++j)
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          const int64_t n = n0 + r * nwarps, k0 = kb + j * 1024 + lane * 32;
          cw[j][r] = make_uint4(0u, 0u, 0u, 0u);
          sw[j][r] = 0;
          if (n < p.N && k0 < K) {
            cw[j][r] = __ldg(reinterpret_cast<const uint4*>(p.codes + n * row_bytes + k0 / 2));
            sw[j][r] = __ldg(reinterpret_cast<const uint16_t*>(p.scales + n * srow_bytes + k0 / 16));
          }
        }
#pragma unroll
      for (int j = 0; j < kJ; ++j) {
        const int64_t k0 = kb + j * 1024 + lane * 32;
        if (k0 < K) step32<kM, kR>(xs4, KC, uint32_t(k0 / 4), cw[j], sw[j], acc);
      }
    }
#pragma unroll
    for (int r = 0; r < kR; ++r) {
      const int64_t n = n0 + r * nwarps;
      float y[kM];
#pragma unroll
      for (int m = 0; m < kM; ++m) {
        y[m] = acc[r][m].x + acc[r][m].y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) y[m] += __shfl_xor_sync(0xFFFFFFFFu, y[m], o);
      }
      if (n < p.N && lane < kM) {
        float a = y[0];
#pragma unroll
        for (int m = 1; m < kM; ++m)
          if (lane == m) a = y[m];
        const float b = p.bias ? __uint_as_float(uint32_t(p.bias[n]) << 16) : 0.0f;
        const __nv_bfloat16 out = __float2bfloat16_rn(fmaf(p.g, a, b));
        p.Y[int64_t(lane) * p.N + n] = *reinterpret_cast<const uint16_t*>(&out);
      }
    }
  }
}

// Blocks per SM for this instance, device and K, queried once (the attribute
// and occupancy calls cost microseconds of host time; a launch should not).
template <int kM>
int blocks_per_sm(int64_t K, size_t smem) {
  static std::atomic<int64_t> cached_key[64];
  static std::atomic<int> cached_val[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int64_t key = K + 1;
  if (cached_key[dev & 63].load() == key) return cached_val[dev & 63].load();
  if (cudaFuncSetAttribute(w4a16_kernel<kM>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, w4a16_kernel<kM>, kThreadsW, smem) != cudaSuccess)
    return 0;
  cached_val[dev & 63].store(per_sm);
  cached_key[dev & 63].store(key);
  return per_sm;
}

template <int kM>
cudaError_t launch_m(const W4A16Params& p, int num_sms, cudaStream_t s) {
  const size_t smem = size_t(kM) * size_t(p.K) * 4;
  const int per_sm = blocks_per_sm<kM>(p.K, smem);
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t rows_per_cta = (kThreadsW / 32) * rows_in_flight<kM>();
  int64_t blocks = int64_t(per_sm) * num_sms;
  const int64_t need = (p.N + rows_per_cta - 1) / rows_per_cta;
  if (blocks > need) blocks = need;
  w4a16_kernel<kM><<<unsigned(blocks), kThreadsW, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w4a16(const W4A16Launch& a, cudaStream_t s, const char** why) {
  W4A16Params p{};
  p.codes = a.layer + a.g.off_codes;
  p.scales = a.layer + a.g.off_scales;
  p.inv_s = reinterpret_cast<const float*>(a.layer + a.g.off_inv_s);
  p.bias = a.has_bias ? reinterpret_cast<const uint16_t*>(a.layer + a.g.off_bias) : nullptr;
  p.K = a.g.K;
  p.N = a.g.N;
  p.g = a.gscale;
  // rows of X in launches of at most kMaxMW, stream ordered
  for (int64_t m0 = 0; m0 < a.M; m0 += kMaxMW) {
    const int64_t mc = a.M - m0 < kMaxMW ? a.M - m0 : kMaxMW;
    p.X = a.X + m0 * a.g.K;
    p.Y = a.Y + m0 * a.g.N;
    p.M = mc;
    cudaError_t e = mc == 1   ? launch_m<1>(p, a.num_sms, s)
                    : mc == 2 ? launch_m<2>(p, a.num_sms, s)
                    : mc == 3 ? launch_m<3>(p, a.num_sms, s)
                              : launch_m<4>(p, a.num_sms, s);
    if (e != cudaSuccess) {
      *why = "launch of the W4A16 kernel failed";
      return e;
    }
  }
  return cudaSuccess;
}

}  // namespace svdq
