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
// in fragment order, so one 16-byte read per lane brings the A operands of
// four MMAs.
//
// A CTA takes 16-row tiles of the output in turn.  One producer thread keeps a
// ring of up to four stages full with bulk copies (cp.async.bulk) of the next
// tiles' codes and scales, up to 48 weight tiles of 16 x 64 (27 KB) per stage,
// so the weight stream never waits for the arithmetic; eight compute warps
// split each row tile's K (tile kt goes to warp kt % 8), read their operands
// from the stage, and add their partial sums through shared memory in a fixed
// order, summed by a warp that rotates with the row tile (the partial-sum
// buffer alternates with the tile, so one barrier per tile suffices).  One row
// of X runs the same MMA path: the MMA is then 7/8 padding, but it does the
// mixed-precision multiply-adds in one instruction per 256 weights, which the
// CUDA cores would spend one instruction per weight on.  Every wait is
// bounded: a timeout sets the layer's status word and the CTA drains its
// copies and exits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>

#include "layout.h"
#include "ptx.cuh"
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

constexpr int kWarpsW = 8;                   // compute warps
constexpr int kThreadsW = 32 * kWarpsW + 32;  // + one producer warp
constexpr int kProducerWarpW = kWarpsW;
constexpr int kMaxMW = 8;  // rows of X per launch: the MMA's N
constexpr int kStagesW = 4;
constexpr uint32_t kTileCodeBytes = 512, kTileScaleBytes = 64;

struct W4A16Params {
  const uint4* codes;   // [N16 / 16][KT][32 lanes] x 16 bytes
  const uint2* scales;  // [N16 / 16][KT][8 groups] x 8 bytes
  const float* inv_s;
  const uint16_t* bias;  // or null
  const uint16_t* X;
  uint16_t* Y;
  uint32_t* status;
  int64_t K, N, M, NT, KT;
  float g;
  int32_t chunk;   // weight tiles (16 x 64) per stage, a multiple of kWarpsW
  int32_t stages;  // ring depth, 2 .. kStagesW
  uint32_t off_red, off_ring, off_ctrl;  // shared-memory sections (bytes)
  uint64_t timeout_ns;
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

// Two bf16 inputs (one word) divided by their s (times 1/s), saturated to f16's range and
// rounded to f16: one word of x~.
__device__ __forceinline__ uint32_t x_tilde2(uint32_t xb, float is_lo, float is_hi) {
  const float lo = fminf(fmaxf(__uint_as_float(xb << 16) * is_lo, -65504.0f), 65504.0f);
  const float hi = fminf(fmaxf(__uint_as_float(xb & 0xFFFF0000u) * is_hi, -65504.0f), 65504.0f);
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Warps 0-7 compute, warp 8 lane 0 fills the ring.  Stage s holds `chunk` weight tiles of
// one row tile: their codes (chunk x 512 bytes), then their scales (chunk x 64 bytes).
__global__ void __launch_bounds__(kThreadsW, 2) w4a16_kernel(const W4A16Params p) {
  extern __shared__ __align__(128) uint8_t smem_w[];
  const int64_t K = p.K;
  const uint32_t RW = uint32_t(K / 2) + 4;  // x~ row stride in f16 pairs (+4: rows start on different banks)
  const uint32_t MR = uint32_t(p.M);        // rows of x~ kept (B columns past M are zero in registers)
  uint32_t* xs = reinterpret_cast<uint32_t*>(smem_w);             // [M][RW] f16 pairs
  float* red = reinterpret_cast<float*>(smem_w + p.off_red);      // [8 warps][32 lanes][4]
  const uint32_t ring_s = ptx::smem_u32(smem_w + p.off_ring);
  const uint32_t stage_bytes = uint32_t(p.chunk) * (kTileCodeBytes + kTileScaleBytes);
  const uint32_t ctrl_s = ptx::smem_u32(smem_w + p.off_ctrl);
  const uint32_t FULL = ctrl_s, EMPTY = ctrl_s + 8u * kStagesW;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem_w + p.off_ctrl + 16u * kStagesW);
  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const int g = lane >> 2, c = lane & 3;
  const int64_t nchunks = (p.KT + p.chunk - 1) / p.chunk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      ptx::mbar_init(FULL + 8u * s, 1);
      ptx::mbar_init(EMPTY + 8u * s, kWarpsW);
    }
    *abort_flag = 0u;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  auto fail = [&](uint32_t code) {
    *abort_flag = 1u;
    atomicOr(p.status, code);
  };

  if (warp == kProducerWarpW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t u = 0;
      bool stop = false;
      for (int64_t nt = blockIdx.x; nt < p.NT && !stop; nt += gridDim.x) {
        for (int64_t ch = 0; ch < nchunks; ++ch, ++u) {
          const uint32_t s = u % uint32_t(p.stages), ph = (u / uint32_t(p.stages)) & 1u;
          if (!ptx::mbar_wait(EMPTY + 8u * s, ph ^ 1u, abort_flag, p.timeout_ns)) {
            fail(0x100u);
            stop = true;
            break;
          }
          const int64_t kt0 = ch * p.chunk;
          const uint32_t n = uint32_t(p.KT - kt0 < p.chunk ? p.KT - kt0 : p.chunk);
          const uint32_t st = ring_s + s * stage_bytes;
          ptx::mbar_expect_tx(FULL + 8u * s, n * (kTileCodeBytes + kTileScaleBytes));
          ptx::bulk_g2s(st, p.codes + (nt * p.KT + kt0) * 32, n * kTileCodeBytes, FULL + 8u * s);
          ptx::bulk_g2s(st + uint32_t(p.chunk) * kTileCodeBytes, p.scales + (nt * p.KT + kt0) * 8,
                        n * kTileScaleBytes, FULL + 8u * s);
        }
      }
      // every issued copy must land before the CTA may exit
      const uint32_t S = uint32_t(p.stages);
      for (uint32_t i = u > S ? u - S : 0; i < u; ++i)
        ptx::mbar_wait(FULL + 8u * (i % S), (i / S) & 1u, nullptr, p.timeout_ns);
    }
    return;  // the compute warps' barriers below count 256 threads
  }

  // ------------------------------------------------------------- compute
  // x~ = f16(x / s), saturating (the producer's first copies are already in flight); eight
  // inputs per thread and step: 16-byte loads (X is 16-byte aligned, K a multiple of 64)
  const uint32_t KV = uint32_t(K / 8);  // 16-byte vectors per row of X
  for (uint32_t i = threadIdx.x; i < MR * KV; i += 32 * kWarpsW) {
    const uint32_t m = i / KV, v = i % KV;
    const uint4 xb = *reinterpret_cast<const uint4*>(p.X + int64_t(m) * K + 8 * int64_t(v));
    const float4 s0 = *reinterpret_cast<const float4*>(p.inv_s + 8 * int64_t(v));
    const float4 s1 = *reinterpret_cast<const float4*>(p.inv_s + 8 * int64_t(v) + 4);
    uint4 o;
    o.x = x_tilde2(xb.x, s0.x, s0.y);
    o.y = x_tilde2(xb.y, s0.z, s0.w);
    o.z = x_tilde2(xb.z, s1.x, s1.y);
    o.w = x_tilde2(xb.w, s1.z, s1.w);
    *reinterpret_cast<uint4*>(xs + m * RW + 4 * v) = o;
  }
  ptx::named_sync(1, 32 * kWarpsW);

  // Every compute warp runs the same loop and meets every barrier, also after a
  // timeout (it then skips the work); only the producer leaves early.
  uint32_t u = 0, tcount = 0;
  bool bad = false;
  for (int64_t nt = blockIdx.x; nt < p.NT; nt += gridDim.x) {
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t* xrow = uint32_t(g) < MR ? xs + uint32_t(g) * RW : nullptr;
    for (int64_t ch = 0; ch < nchunks; ++ch, ++u) {
      const uint32_t s = u % uint32_t(p.stages), ph = (u / uint32_t(p.stages)) & 1u;
      if (!bad) {
        bool ok = ptx::mbar_wait(FULL + 8u * s, ph, abort_flag, p.timeout_ns);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0 && *abort_flag == 0u) fail(0x200u);
          bad = true;
        }
      }
      if (!bad) {
        const int64_t kt0 = ch * p.chunk;
        const int n = int(p.KT - kt0 < p.chunk ? p.KT - kt0 : p.chunk);
        const uint8_t* st = smem_w + p.off_ring + s * stage_bytes;
        const uint4* cws = reinterpret_cast<const uint4*>(st);
        const uint2* sws = reinterpret_cast<const uint2*>(st + uint32_t(p.chunk) * kTileCodeBytes);
        for (int i = warp; i < n; i += kWarpsW) {
          const uint32_t kt = uint32_t(kt0) + uint32_t(i);
          const uint4 cw = cws[i * 32 + lane];
          const uint2 sw = sws[i * 8 + g];
          tile_mma(acc, cw, sw, xrow ? xrow + kt * 32u : nullptr, c);
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(EMPTY + 8u * s);  // this warp is done with the stage
      }
    }
    // the 8 warps' partial tiles, added in warp order by one warp (rotating); the buffer
    // alternates with the row tile, so one barrier per tile suffices
    float* rb = red + (tcount & 1u) * (kWarpsW * 32 * 4);
    *reinterpret_cast<float4*>(rb + (warp * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    ptx::named_sync(1, 32 * kWarpsW);
    if (warp == int(tcount % kWarpsW) && !bad) {
      float4 t = *reinterpret_cast<const float4*>(rb + lane * 4);
#pragma unroll
      for (int w = 1; w < kWarpsW; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(rb + (w * 32 + lane) * 4);
        t.x += v.x;
        t.y += v.y;
        t.z += v.z;
        t.w += v.w;
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
    ++tcount;
  }
}

// Blocks per SM for this device and shared-memory size, queried once (the
// attribute and occupancy calls cost microseconds of host time; a launch
// should not).  The carveout asks for all of the unified L1 as shared memory,
// or the driver may size it for one CTA.
int blocks_per_sm(size_t smem) {
  static std::atomic<int64_t> cached_key[64];
  static std::atomic<int> cached_val[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int64_t key = int64_t(smem) + 1;
  if (cached_key[dev & 63].load() == key) return cached_val[dev & 63].load();
  if (cudaFuncSetAttribute(w4a16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess ||
      cudaFuncSetAttribute(w4a16_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           int(cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
    return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, w4a16_kernel, kThreadsW, smem) != cudaSuccess)
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
  p.status = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.layer));  // the image's first word
  p.K = a.g.K;
  p.N = a.g.N;
  p.NT = a.g.N16 / 16;
  p.KT = a.g.KT;
  p.g = a.gscale;
  p.timeout_ns = a.timeout_ns;
  // rows of X in launches of at most 8 (the MMA's N), stream ordered
  for (int64_t m0 = 0; m0 < a.M; m0 += kMaxMW) {
    p.X = a.X + m0 * a.g.K;
    p.Y = a.Y + m0 * a.g.N;
    p.M = a.M - m0 < kMaxMW ? a.M - m0 : kMaxMW;
    // shared memory: x~ | partial sums | ring | barriers.  Two CTAs per SM if a ring of two
    // or more stages (40 KB or more, or all of K) fits in half the SM, else one CTA; the
    // largest stage first.
    const size_t xs_bytes = size_t(round_up(int64_t(p.M) * (a.g.K / 2 + 4) * 4, 128));
    const size_t red_bytes = 2 * size_t(kWarpsW) * 32 * 16, ctrl_bytes = 128;
    const size_t fixed = xs_bytes + red_bytes + ctrl_bytes;
    const int64_t max_chunk = round_up(p.KT, kWarpsW);
    size_t smem = 0;
    for (size_t budget : {size_t(113) * 1024, size_t(227) * 1024}) {
      for (int64_t chunk = 48; chunk >= kWarpsW && smem == 0; chunk -= kWarpsW) {
        const int64_t ck = chunk < max_chunk ? chunk : max_chunk;
        const size_t stage = size_t(ck) * (kTileCodeBytes + kTileScaleBytes);
        if (fixed + 2 * stage > budget) continue;
        int64_t st = int64_t((budget - fixed) / stage);
        if (st > kStagesW) st = kStagesW;
        // two CTAs per SM only with at least 40 KB of weights in flight per CTA
        if (budget < size_t(227) * 1024 && size_t(st) * stage < size_t(40) * 1024 && ck < max_chunk) continue;
        p.chunk = int32_t(ck);
        p.stages = int32_t(st);
        smem = fixed + size_t(st) * stage;
      }
      if (smem) break;
    }
    if (smem == 0) {
      *why = "K is too large for the W4A16 kernel (x~ leaves no room for its weight ring)";
      return cudaErrorInvalidConfiguration;
    }
    p.off_red = uint32_t(xs_bytes);
    p.off_ring = uint32_t(xs_bytes + red_bytes);
    p.off_ctrl = uint32_t(xs_bytes + red_bytes + size_t(p.stages) * size_t(p.chunk) * (kTileCodeBytes + kTileScaleBytes));
    const int per_sm = blocks_per_sm(smem);
    if (per_sm < 1) {
      *why = "the W4A16 kernel does not fit on this device";
      return cudaErrorInvalidConfiguration;
    }
    int64_t blocks = int64_t(per_sm) * a.num_sms;
    if (blocks > p.NT) blocks = p.NT;
    w4a16_kernel<<<unsigned(blocks), kThreadsW, smem, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      *why = "launch of the W4A16 kernel failed";
      return e;
    }
  }
  return cudaSuccess;
}

}  // namespace svdq
