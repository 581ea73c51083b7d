// act_quant.cu -- kernel 1: smoothing, NVFP4 quantization and low-rank down projection of X
// in one pass over X.
//
// SVDQuant summary page, section 4.3 "Nunchaku" (Figure 6(b)): the down
// projection of the low-rank branch shares the activation read of the
// quantization kernel, so X leaves HBM once.  Per 16 elements along K:
//   x_hat = bf16(x * (1/lambda))                           (section 4.2 smoothing)
//   s_b   = E4M3(amax|x_hat| * c_a),  c_a = 1 / (6 g_a)     (section 3 quantizer,
//   d     = value(s_b) * g_a,  code = E2M1(x_hat * rcp(d))   q_max = 6, per block)
// and lr' = bf16((x_hat L1) / (g_a g_w)) on the tensor cores.
//
// Design (sm_100a):
//   * CTA = 128 rows of X x a slice of K.  The producer warp streams X chunks
//     of 128 rows x 64 columns with a 2D TMA load (128-byte swizzle), the
//     matching 1/lambda slice and L1^T chunk with bulk copies, through an
//     mbarrier ring (4 stages with two CTAs per SM, 6 or 8 with one).
//   * Converter warps (one group of 8 with two CTAs per SM, two groups taking
//     alternate chunks with one): two threads per row convert 32 elements
//     each in shared memory, write x_hat back in place (it is the A operand
//     of the MMA), and store codes and block scales straight into the GEMM's
//     tiled layout.
//   * The MMA warp: one thread issues tcgen05.mma kind::f16 (M = 128,
//     N = rank) accumulating X_hat L1 in tensor memory.
//   * K is split across the CTAs of a cluster so that enough CTAs stream HBM;
//     their partial X_hat L1 tiles are summed in a fixed order through
//     distributed shared memory (no global scratch, deterministic).
//   * Every wait is bounded; a timeout sets the layer's status word and the
//     CTA drains its copies and MMAs, frees tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <map>
#include <mutex>
#include <tuple>

#include "kernels.h"
#include "ptx.cuh"

namespace svdq {

namespace {

using namespace ptx;

// S stages and G groups of eight converter warps (group g takes the chunks i with i % G == g),
// then the producer warp and the MMA warp.  S = 4 has one group and runs two CTAs per SM; the
// one-CTA-per-SM instances (S = 6 or 8) have two groups, and S is even, so that a stage's chunks
// always belong to one group.
constexpr int kConvThreads = 256;  // one group
__host__ __device__ constexpr int groups1(int stages) { return stages == 4 ? 1 : 2; }
__host__ __device__ constexpr int threads1(int stages) { return 32 * (8 * groups1(stages) + 2); }
constexpr uint32_t ctrl_bytes1(int stages) { return 32u * uint32_t(stages) + 512u; }  // barriers + reciprocal table
constexpr int kMaxSplits = 8;       // pulled partials: a portable cluster
constexpr int kMaxPushSplits = 16;  // pushed partials: up to the non-portable cluster size
constexpr uint32_t kXBytes = kBM * 128;  // 16 KB: 128 rows x 64 bf16
constexpr uint32_t kInvSlot = 1024;      // 64 floats of 1/lambda (256 B), padded for alignment

struct ActQuantParams {
  const float* inv_lam;  // [KC * 64]
  const uint8_t* l1t;    // L1^T chunks, rc16 rows of 128 B each
  uint8_t* codes;        // act + off_codes
  uint8_t* sf;           // act + off_sf
  uint8_t* lr;           // act + off_lr
  uint32_t* status;      // layer status word
  int32_t MT, KT, KC, RJ, r_tot, rc16, splits;
  int32_t push;          // split partials are pushed to the owning CTA (else pulled)
  int32_t rows_per;      // rows of a row tile each CTA of the cluster reduces
  uint32_t stage_bytes, tmem_cols, rb_bytes;
  float g_a, c_a, inv_alpha;
  uint64_t timeout_ns;
};

// One 16-element block of one row: read x from the swizzled stage, write
// x_hat back, return 8 bytes of E2M1 codes and the E4M3 block scale.
__device__ __forceinline__ void quant_block(uint8_t* xrow, uint32_t t7, int g, const float* inv, const float* rtab,
                                            float c_a, bool write_back, uint32_t& w0, uint32_t& w1,
                                            uint32_t& scale) {
  uint4* p0 = reinterpret_cast<uint4*>(xrow + (((2u * g) ^ t7) << 4));
  uint4* p1 = reinterpret_cast<uint4*>(xrow + (((2u * g + 1u) ^ t7) << 4));
  const uint4 a = *p0, b = *p1;
  const float4* iv = reinterpret_cast<const float4*>(inv);
  const float4 i0 = iv[0], i1 = iv[1], i2 = iv[2], i3 = iv[3];
  const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  const float il[16] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w,
                        i2.x, i2.y, i2.z, i2.w, i3.x, i3.y, i3.z, i3.w};
  uint32_t h[8];
  float xh[16];
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float lo = __fmul_rn(bf16lo(in[j]), il[2 * j]);
    const float hi = __fmul_rn(bf16hi(in[j]), il[2 * j + 1]);
    h[j] = f32x2_to_bf16x2(lo, hi);
    xh[2 * j] = bf16lo(h[j]);
    xh[2 * j + 1] = bf16hi(h[j]);
    amax = fmaxf(amax, fmaxf(fabsf(xh[2 * j]), fabsf(xh[2 * j + 1])));
  }
  if (write_back) {  // x_hat is the A operand of the down projection
    *p0 = make_uint4(h[0], h[1], h[2], h[3]);
    *p1 = make_uint4(h[4], h[5], h[6], h[7]);
  }
  const uint32_t sc = f32_to_e4m3(__fmul_rn(amax, c_a));
  const float rcp = rtab[sc];
  w0 = f32x8_to_e2m1(__fmul_rn(xh[0], rcp), __fmul_rn(xh[1], rcp), __fmul_rn(xh[2], rcp), __fmul_rn(xh[3], rcp),
                     __fmul_rn(xh[4], rcp), __fmul_rn(xh[5], rcp), __fmul_rn(xh[6], rcp), __fmul_rn(xh[7], rcp));
  w1 = f32x8_to_e2m1(__fmul_rn(xh[8], rcp), __fmul_rn(xh[9], rcp), __fmul_rn(xh[10], rcp),
                     __fmul_rn(xh[11], rcp), __fmul_rn(xh[12], rcp), __fmul_rn(xh[13], rcp),
                     __fmul_rn(xh[14], rcp), __fmul_rn(xh[15], rcp));
  scale = sc;
}

// INT4 instance: the smoothing half of quant_block for one 16-element block:
// x_hat (bf16 values, as floats) into xh, written back in place when asked,
// and the running amax of the block.
__device__ __forceinline__ void smooth_block(uint8_t* xrow, uint32_t t7, int g, const float* inv, bool write_back,
                                             float* xh, float& amax) {
  uint4* p0 = reinterpret_cast<uint4*>(xrow + (((2u * g) ^ t7) << 4));
  uint4* p1 = reinterpret_cast<uint4*>(xrow + (((2u * g + 1u) ^ t7) << 4));
  const uint4 a = *p0, b = *p1;
  const float4* iv = reinterpret_cast<const float4*>(inv);
  const float4 i0 = iv[0], i1 = iv[1], i2 = iv[2], i3 = iv[3];
  const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  const float il[16] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w,
                        i2.x, i2.y, i2.z, i2.w, i3.x, i3.y, i3.z, i3.w};
  uint32_t h[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float lo = __fmul_rn(bf16lo(in[j]), il[2 * j]);
    const float hi = __fmul_rn(bf16hi(in[j]), il[2 * j + 1]);
    h[j] = f32x2_to_bf16x2(lo, hi);
    xh[2 * j] = bf16lo(h[j]);
    xh[2 * j + 1] = bf16hi(h[j]);
    amax = fmaxf(amax, fmaxf(fabsf(xh[2 * j]), fabsf(xh[2 * j + 1])));
  }
  if (write_back) {
    *p0 = make_uint4(h[0], h[1], h[2], h[3]);
    *p1 = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// Eight INT4 codes q = clamp(rne(x * rcp), -7, 7) as two's-complement nibbles,
// element 0 in the low nibble.
__device__ __forceinline__ uint32_t int4x8(const float* x, float rcp) {
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int q = min(7, max(-7, __float2int_rn(__fmul_rn(x[j], rcp))));
    w |= (uint32_t(q) & 0xFu) << (4 * j);
  }
  return w;
}

// Scale 8 fp32 ranks by 1/alpha, round to bf16, store 16 bytes of lr'.
__device__ __forceinline__ void store_lr8(const ActQuantParams& p, int mt, uint32_t row, int c, const float* v) {
  uint4 w;
  w.x = f32x2_to_bf16x2(__fmul_rn(v[0], p.inv_alpha), __fmul_rn(v[1], p.inv_alpha));
  w.y = f32x2_to_bf16x2(__fmul_rn(v[2], p.inv_alpha), __fmul_rn(v[3], p.inv_alpha));
  w.z = f32x2_to_bf16x2(__fmul_rn(v[4], p.inv_alpha), __fmul_rn(v[5], p.inv_alpha));
  w.w = f32x2_to_bf16x2(__fmul_rn(v[6], p.inv_alpha), __fmul_rn(v[7], p.inv_alpha));
  uint8_t* tile = p.lr + (size_t(mt) * p.RJ + size_t(c / kRChunk)) * kATileBytes;
  *reinterpret_cast<uint4*>(tile + sw128(row, uint32_t(c % kRChunk) * 2u)) = w;
}

// kLowRank = false (rank 0) leaves out every tensor-core instruction: a kernel
// that allocates tensor memory runs one CTA per SM, the plain quantizer two.
// kInt4 selects the INT4 quantizer (groups of 64, bf16 scales) for the NVFP4 one;
// the smoothing, the down projection and its reduction are the same.
template <bool kLowRank, bool kInt4 = false, int kS = 4>
__global__ void __launch_bounds__(threads1(kS), kS == 4 ? 2 : 1)
    act_quant_kernel(const __grid_constant__ CUtensorMap tmap_x, const ActQuantParams p) {
  constexpr int kG = groups1(kS);
  static_assert(kS % kG == 0, "a stage's chunks must belong to one converter group");
  constexpr int kProducerWarp1 = 8 * kG, kMmaWarp1 = 8 * kG + 1;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;

  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const int split = int(blockIdx.x), mt = int(blockIdx.y);
  const int kc0 = int(int64_t(split) * p.KC / p.splits);
  const int kc1 = int(int64_t(split + 1) * p.KC / p.splits);
  const int nchunks = kc1 - kc0;
  constexpr bool lowrank = kLowRank;

  // [stages][receive buffer of pushed partials: splits x rows_per x r_tot floats][control]
  const uint32_t rb_s = sbase + kS * p.stage_bytes;
  const float* rb = reinterpret_cast<const float*>(smem + kS * p.stage_bytes);
  uint8_t* ctrl = smem + kS * p.stage_bytes + p.rb_bytes;
  const uint32_t ctrl_s = sbase + kS * p.stage_bytes + p.rb_bytes;
  // control block: FULL, CONV, EMPTY [kS] each, ACCF, DRAIN, the tensor-memory slot, the abort
  // flag, RECV; the block-reciprocal table at 32 kS
  constexpr uint32_t kB = 8u * kS;
  const uint32_t FULL = ctrl_s, CONV = ctrl_s + kB, EMPTY = ctrl_s + 2u * kB;
  const uint32_t ACCF = ctrl_s + 3u * kB, DRAIN = ACCF + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 3u * kB + 16u);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(ctrl + 3u * kB + 20u);
  const uint32_t RECV = ctrl_s + 3u * kB + 24u;  // the pushed partials of this CTA's rows have landed
  float* rtab = reinterpret_cast<float*>(ctrl + 4u * kB);
  const int crank = kLowRank && p.splits > 1 ? int(cluster_ctarank()) : 0;
  const int own0 = crank * p.rows_per;
  const int own1 = own0 + p.rows_per < kBM ? own0 + p.rows_per : kBM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kS; ++s) {
      mbar_init(FULL + 8u * s, 1);
      mbar_init(CONV + 8u * s, kConvThreads);
      mbar_init(EMPTY + 8u * s, 1);
    }
    mbar_init(ACCF, 1);
    mbar_init(DRAIN, 1);
    mbar_init(RECV, 1);
    *abort_flag = 0u;
    if (lowrank && p.push)  // every CTA of the cluster pushes its partial of these rows
      mbar_expect_tx(RECV, uint32_t(p.splits * (own1 - own0) * p.r_tot * 4));
    fence_mbar_init();
  }
  // 1 / d for every block-scale code s (d = value(s) g_a, g_a static; 0 where d is 0): one
  // shared-memory load per block instead of decoding s and a correctly rounded reciprocal
  if (threadIdx.x < 128) {
    const float d = __fmul_rn(e4m3_value(threadIdx.x), p.g_a);
    rtab[threadIdx.x] = (d == 0.0f || threadIdx.x == 127u) ? 0.0f : __frcp_rn(d);
  }
  if (warp == kMmaWarp1 && lowrank) {
    tmem_alloc(ctrl_s + 3u * kB + 16u, p.tmem_cols);
    tmem_relinquish();
  }
  if (lowrank) tc_fence_before();
  __syncthreads();
  if (lowrank) tc_fence_after();
  const uint32_t tmem = lowrank ? *tmem_slot : 0u;
  // the receive barriers of the whole cluster are armed before anyone pushes
  if (lowrank && p.push) cluster_arrive();
  // X may be the previous kernel's output and the activation buffer its input
  griddep_wait();
  griddep_launch_dependents();

  auto fail = [&](uint32_t code) {
    *abort_flag = 1u;
    atomicOr(p.status, code);
  };

  if (warp == kProducerWarp1) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmap_x);
      const uint32_t tx = kXBytes + 256u + (lowrank ? uint32_t(p.r_tot) * 128u : 0u);
      int issued = 0;
      for (int i = 0; i < nchunks; ++i) {
        const int s = i % kS;
        const uint32_t ph = uint32_t(i / kS) & 1u;
        if (!mbar_wait(EMPTY + 8u * s, ph ^ 1u, abort_flag, p.timeout_ns)) {
          fail(0x1u);
          break;
        }
        const uint32_t st = sbase + uint32_t(s) * p.stage_bytes;
        const int kc = kc0 + i;
        mbar_expect_tx(FULL + 8u * s, tx);
        tma_load_2d(st, &tmap_x, kc * kKChunk, mt * kBM, FULL + 8u * s);
        bulk_g2s(st + kXBytes, p.inv_lam + size_t(kc) * kKChunk, 256u, FULL + 8u * s);
        if (lowrank)
          bulk_g2s(st + kXBytes + kInvSlot, p.l1t + size_t(kc) * size_t(p.rc16) * 128u, uint32_t(p.r_tot) * 128u,
                   FULL + 8u * s);
        issued = i + 1;
      }
      // every issued copy must land before this CTA may exit
      for (int i = issued > kS ? issued - kS : 0; i < issued; ++i)
        mbar_wait(FULL + 8u * (i % kS), uint32_t(i / kS) & 1u, nullptr, p.timeout_ns);
    }
    __syncwarp();
  } else if (kInt4 && warp < 8 * kG) {
    // ------------------------------------------------------ INT4 converters
    // two threads per row, neighbours in a warp: thread (t, h) converts
    // elements 32 h .. 32 h + 31 of row t; the chunk is one group of 64, whose
    // amax the pair shares
    const uint32_t t = uint32_t(warp & 7) * 16u + (uint32_t(lane) >> 1), h = uint32_t(lane) & 1u;
    const uint32_t t7 = t & 7u;
    for (int i = warp >> 3; i < nchunks; i += kG) {
      const int s = i % kS;
      const uint32_t ph = uint32_t(i / kS) & 1u;
      bool ok = mbar_wait(FULL + 8u * s, ph, abort_flag, p.timeout_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);  // the pair's shuffle below needs the whole warp
      if (!ok) {
        if (lane == 0) fail(0x2u);
        break;
      }
      uint8_t* stage = smem + size_t(s) * p.stage_bytes;
      uint8_t* xrow = stage + t * 128u;
      const float* inv = reinterpret_cast<const float*>(stage + kXBytes);
      float xh[32];
      float amax = 0.0f;
      smooth_block(xrow, t7, int(2 * h), inv + 32 * h, lowrank, xh, amax);
      smooth_block(xrow, t7, int(2 * h + 1), inv + 32 * h + 16, lowrank, xh + 16, amax);
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      const uint32_t sb = f32x2_to_bf16x2(__fdiv_rn(amax, 7.0f), 0.0f) & 0xFFFFu;  // s = bf16(amax / 7)
      const float sv = __uint_as_float(sb << 16);
      const float rcp = sv == 0.0f ? 0.0f : __frcp_rn(sv);
      const uint4 cw = make_uint4(int4x8(xh, rcp), int4x8(xh + 8, rcp), int4x8(xh + 16, rcp), int4x8(xh + 24, rcp));
      const int kc = kc0 + i;
      const size_t blk = size_t(mt) * p.KC + size_t(kc);
      *reinterpret_cast<uint4*>(p.codes + blk * 4096u + h * 2048u + t * 16u) = cw;
      if (h == 0) *reinterpret_cast<uint16_t*>(p.sf + (blk * 128u + t) * 2u) = uint16_t(sb);
      if (lowrank) fence_proxy_async_smem();  // x_hat (generic writes) -> tensor-core reads
      mbar_arrive(CONV + 8u * s);
    }
  } else if (warp < 8 * kG) {
    // ----------------------------------------------------------- converters
    // two threads per row: thread (t, h) converts elements 32 h .. 32 h + 31
    // of row t of each 64-column chunk (two 16-element blocks)
    const uint32_t t = threadIdx.x & 127u, h = (threadIdx.x >> 7) & 1u;
    const uint32_t t7 = t & 7u;
    for (int i = warp >> 3; i < nchunks; i += kG) {
      const int s = i % kS;
      const uint32_t ph = uint32_t(i / kS) & 1u;
      if (!mbar_wait(FULL + 8u * s, ph, abort_flag, p.timeout_ns)) {
        fail(0x2u);
        break;
      }
      uint8_t* stage = smem + size_t(s) * p.stage_bytes;
      uint8_t* xrow = stage + t * 128u;
      const float* inv = reinterpret_cast<const float*>(stage + kXBytes);
      uint32_t cw[4], sc[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int g = int(2 * h) + j;
        quant_block(xrow, t7, g, inv + 16 * g, rtab, p.c_a, lowrank, cw[2 * j],
                    cw[2 * j + 1], sc[j]);
      }
      const int kc = kc0 + i, kt = kc >> 2, sub = kc & 3;
      uint8_t* ctile = p.codes + (size_t(mt) * p.KT + kt) * kATileBytes;
      *reinterpret_cast<uint4*>(ctile + sw128(t, uint32_t(sub) * 32u + h * 16u)) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      uint8_t* stile = p.sf + (size_t(mt) * p.KT + kt) * kSFATileBytes + size_t(sub) * kSFAtomBytes;
      *reinterpret_cast<uint16_t*>(stile + sf_atom(t, 2u * h)) = uint16_t(sc[0] | (sc[1] << 8));
      if (lowrank) fence_proxy_async_smem();  // x_hat (generic writes) -> tensor-core reads
      mbar_arrive(CONV + 8u * s);
    }
  } else if (warp == kMmaWarp1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      bool any = false;
      const uint32_t idesc = idesc_bf16(p.r_tot);
      for (int i = 0; i < nchunks; ++i) {
        const int s = i % kS;
        const uint32_t ph = uint32_t(i / kS) & 1u;
        if (!mbar_wait(CONV + 8u * s, ph, abort_flag, p.timeout_ns)) {
          fail(0x4u);
          break;
        }
        if (lowrank) {
          if (!mbar_wait(FULL + 8u * s, ph, abort_flag, p.timeout_ns)) {
            fail(0x4u);
            break;
          }
          tc_fence_after();
          const uint32_t xa = sbase + uint32_t(s) * p.stage_bytes;
          const uint32_t la = xa + kXBytes + kInvSlot;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            umma_bf16(tmem, sdesc_sw128(xa + 32u * ks), sdesc_sw128(la + 32u * ks), idesc, (i | ks) ? 1u : 0u);
          tc_commit(EMPTY + 8u * s);
          any = true;
        } else {
          mbar_arrive(EMPTY + 8u * s);
        }
      }
      if (any) {
        tc_commit(ACCF);
        tc_commit(DRAIN);
        mbar_wait(DRAIN, 0u, nullptr, p.timeout_ns);
      }
    }
    __syncwarp();
  }

  // ------------------------------------------------- low-rank output lr'
  if (lowrank && p.push) {
    // each thread of warps 0-3 holds one row's float partial; it goes to the
    // CTA of the cluster that reduces that row, which adds the splits in order
    if (warp < 4) {
      bool ok = (*abort_flag == 0u) && mbar_wait(ACCF, 0u, abort_flag, p.timeout_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      cluster_wait();
      if (ok) {
        tc_fence_after();
        const uint32_t t = threadIdx.x;
        const uint32_t owner = t / uint32_t(p.rows_per), lrow = t % uint32_t(p.rows_per);
        const uint32_t dst = mapa(rb_s + uint32_t(((crank * p.rows_per) + int(lrow)) * p.r_tot) * 4u, owner);
        const uint32_t bar = mapa(RECV, owner);
        const uint32_t taddr = tmem + (uint32_t(warp * 32) << 16);
        for (int c = 0; c < p.r_tot; c += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + uint32_t(c), v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_async_v4(dst + uint32_t(c + 4 * j) * 4u,
                        make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                    __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])),
                        bar);
        }
      } else if (*abort_flag == 0u) {
        fail(0x8u);
      }
    }
    if (warp < 8) {
      bool ok = mbar_wait(RECV, 0u, abort_flag, p.timeout_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0 && *abort_flag == 0u) fail(0x8u);
      } else {
        const int groups = p.r_tot / 4;
        const int nrows = own1 - own0;
        for (int item = int(threadIdx.x); item < nrows * groups; item += kConvThreads) {
          const int lr = item / groups, c = (item % groups) * 4;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int q = 0; q < p.splits; ++q) {  // fixed order: deterministic sums
            const float4 v = *reinterpret_cast<const float4*>(rb + size_t((q * p.rows_per + lr) * p.r_tot + c));
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
          }
          uint2 w;
          w.x = f32x2_to_bf16x2(__fmul_rn(acc.x, p.inv_alpha), __fmul_rn(acc.y, p.inv_alpha));
          w.y = f32x2_to_bf16x2(__fmul_rn(acc.z, p.inv_alpha), __fmul_rn(acc.w, p.inv_alpha));
          uint8_t* tile = p.lr + (size_t(mt) * p.RJ + size_t(c / kRChunk)) * kATileBytes;
          *reinterpret_cast<uint2*>(tile + sw128(uint32_t(own0 + lr), uint32_t(c % kRChunk) * 2u)) = w;
        }
      }
    }
  } else if (lowrank) {
    const bool multi = p.splits > 1;
    float* part = reinterpret_cast<float*>(smem);  // stages are idle now: [128][r_tot + 4]
    const int pstride = p.r_tot + 4;
    if (warp < 4) {
      bool ok = (*abort_flag == 0u) && mbar_wait(ACCF, 0u, abort_flag, p.timeout_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (ok) {
        tc_fence_after();
        const uint32_t t = threadIdx.x;
        const uint32_t taddr = tmem + (uint32_t(warp * 32) << 16);
        for (int c = 0; c < p.r_tot; c += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + uint32_t(c), v);
          tmem_wait_ld();
          float f[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) f[j] = __uint_as_float(v[j]);
          if (multi) {
            float4* dst = reinterpret_cast<float4*>(part + size_t(t) * pstride + c);
            dst[0] = make_float4(f[0], f[1], f[2], f[3]);
            dst[1] = make_float4(f[4], f[5], f[6], f[7]);
            dst[2] = make_float4(f[8], f[9], f[10], f[11]);
            dst[3] = make_float4(f[12], f[13], f[14], f[15]);
          } else {
            store_lr8(p, mt, t, c, f);
            store_lr8(p, mt, t, c + 8, f + 8);
          }
        }
      } else if (*abort_flag == 0u) {
        fail(0x8u);
      }
    }
    if (multi) {
      cluster_sync();  // every partial tile of the cluster is in shared memory
      if (warp < 8 && *abort_flag == 0u) {
        // this CTA sums rows [row0, row1) over the cluster, 4 ranks per item;
        // all peer loads of an item are in flight before the (ordered) adds
        const int rows = (kBM + p.splits - 1) / p.splits;
        const int rank = int(cluster_ctarank());
        const int row0 = rank * rows;
        const int row1 = row0 + rows < kBM ? row0 + rows : kBM;
        const int groups = p.r_tot / 4;
        for (int item = int(threadIdx.x); item < (row1 - row0) * groups; item += kConvThreads) {
          const int row = row0 + item / groups, c = (item % groups) * 4;
          const uint32_t local = sbase + uint32_t((row * pstride + c) * 4);
          float4 v[kMaxSplits];
#pragma unroll
          for (int q = 0; q < kMaxSplits; ++q)
            if (q < p.splits) v[q] = ld_dsmem_f4(mapa(local, uint32_t(q)));
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int q = 0; q < kMaxSplits; ++q)  // fixed order: deterministic sums
            if (q < p.splits) {
              acc.x += v[q].x;
              acc.y += v[q].y;
              acc.z += v[q].z;
              acc.w += v[q].w;
            }
          uint2 w;
          w.x = f32x2_to_bf16x2(__fmul_rn(acc.x, p.inv_alpha), __fmul_rn(acc.y, p.inv_alpha));
          w.y = f32x2_to_bf16x2(__fmul_rn(acc.z, p.inv_alpha), __fmul_rn(acc.w, p.inv_alpha));
          uint8_t* tile = p.lr + (size_t(mt) * p.RJ + size_t(c / kRChunk)) * kATileBytes;
          *reinterpret_cast<uint2*>(tile + sw128(uint32_t(row), uint32_t(c % kRChunk) * 2u)) = w;
        }
      }
      cluster_sync();  // peers keep their shared memory until every read is done
    }
  }

  // ------------------------------------------------------------ teardown
  if (lowrank) tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp1 && lowrank) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

uint32_t next_pow2_at_least32(int v) {
  uint32_t c = 32;
  while (c < uint32_t(v)) c <<= 1;
  return c;
}

}  // namespace

cudaError_t launch_act_quant(const ActQuantLaunch& a, cudaStream_t s, const char** why) {
  const LayerGeom& lg = a.lg;
  const ActGeom ag = make_act_geom(lg, a.M);
  if (ag.MT > 65535) {
    *why = "M too large for one launch (more than 65535 tiles of 128 rows)";
    return cudaErrorInvalidValue;
  }
  auto encode = tensor_map_encoder();
  if (!encode) {
    *why = "cuTensorMapEncodeTiled is not available from the driver";
    return cudaErrorNotSupported;
  }
  alignas(64) CUtensorMap map;
  const cuuint64_t dims[2] = {cuuint64_t(lg.K), cuuint64_t(a.M)};
  const cuuint64_t strides[1] = {cuuint64_t(lg.K) * 2u};
  const cuuint32_t box[2] = {uint32_t(kKChunk), uint32_t(kBM)};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult cr = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.X), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    *why = "cuTensorMapEncodeTiled rejected the X operand";
    return cudaErrorInvalidValue;
  }

  ActQuantParams p{};
  p.inv_lam = reinterpret_cast<const float*>(a.layer + lg.off_inv_lam);
  p.l1t = a.layer + lg.off_l1t;
  p.codes = a.act + ag.off_codes;
  p.sf = a.act + ag.off_sf;
  p.lr = a.act + ag.off_lr;
  p.status = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.layer) + lg.off_status);
  p.MT = int32_t(ag.MT);
  p.KT = int32_t(lg.KT);
  p.KC = int32_t(lg.KC);
  p.RJ = int32_t(lg.RJ);
  p.r_tot = a.r_tot;
  p.rc16 = int32_t(lg.RC16);
  p.stage_bytes = uint32_t(round_up(kXBytes + kInvSlot + uint32_t(a.r_tot) * 128u, 1024));
  p.tmem_cols = a.r_tot > 0 ? next_pow2_at_least32(a.r_tot) : 0u;
  p.g_a = a.g_a;
  p.c_a = a.c_a;
  p.inv_alpha = a.inv_alpha;
  p.timeout_ns = a.timeout_ns;

  const bool lowrank = a.r_tot > 0;
  int dev = 0;
  cudaGetDevice(&dev);
  auto set_smem = [&](auto k, int which, size_t bytes) -> cudaError_t {
    // the attributes are per device and kernel: remember the largest size set on each
    static std::atomic<size_t> smem_set[8][64];
    std::atomic<size_t>& done = smem_set[which][dev & 63];
    if (bytes <= done.load()) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
    if (e == cudaSuccess)  // all of the unified L1 as shared memory: two CTAs per SM must fit
      e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared));
    if (e == cudaSuccess) done.store(bytes);
    return e;
  };
  // Split count: enough CTAs to fill the GPU, then (low rank) the largest cluster
  // size whose clusters of the row tiles are all resident at once.  Occupancy
  // is asked of the rank-0 instance, which has the same resources but no
  // tensor-memory allocation (for which the calculator assumes one CTA per SM,
  // while clusters of this kernel run two per SM).
  auto plan = [&](int sp, int stages, size_t* smem_out, int* push_out, int* rows_out, uint32_t* rb_out) {
    const int rows = (kBM + sp - 1) / sp;
    const size_t base = size_t(stages) * p.stage_bytes + ctrl_bytes1(stages) + 1024;
    const size_t rb = lowrank && sp > 1 ? size_t(round_up(int64_t(sp) * rows * a.r_tot * 4, 1024)) : 0;
    const bool push = rb > 0 && (base + rb <= 113 * 1024 || (base > 113 * 1024 && base + rb <= 227 * 1024));
    *push_out = push ? 1 : 0;
    *rows_out = rows;
    *rb_out = push ? uint32_t(rb) : 0u;
    *smem_out = base + (push ? rb : 0);
  };
  size_t smem = 0;
  int push = 0, rows_per = kBM;
  uint32_t rb_bytes = 0;
  // the split count is planned once per device and shape (it queries the runtime's cluster occupancy)
  using PlanKey = std::tuple<int, int64_t, int32_t, int32_t, int>;
  static std::mutex plan_mu;
  // split count, stages, least shared memory
  static std::map<PlanKey, std::tuple<int, int, size_t>> planned;
  const PlanKey key{dev, ag.MT, p.KC, a.r_tot, a.num_sms};
  int cached = 0, stages = 4;
  size_t min_smem = 0;
  {
    std::lock_guard<std::mutex> lk(plan_mu);
    auto it = planned.find(key);
    if (it != planned.end()) std::tie(cached, stages, min_smem) = it->second;
  }
  plan(1, 4, &smem, &push, &rows_per, &rb_bytes);
  const int per_sm = smem <= 113 * 1024 ? 2 : 1;
  int splits = cached > 0 ? cached : int((int64_t(per_sm) * a.num_sms) / ag.MT);
  const int max_splits = lowrank ? kMaxPushSplits : 64;
  if (splits > max_splits) splits = max_splits;
  if (splits > p.KC) splits = p.KC;
  if (splits < 1) splits = 1;
  if (lowrank && cached == 0) {
    static std::atomic<int> nonportable[64];
    if (nonportable[dev & 63].load() == 0) {
      // clusters of up to 16 CTAs for the pushed partials (small M, long K)
      cudaError_t e = cudaFuncSetAttribute(act_quant_kernel<false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(act_quant_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(act_quant_kernel<true, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(act_quant_kernel<true, false, 8>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(act_quant_kernel<true, true, 8>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(act_quant_kernel<true, false, 6>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(act_quant_kernel<true, true, 6>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      nonportable[dev & 63].store(e == cudaSuccess ? 1 : -1);
    }
    const int cap = nonportable[dev & 63].load() > 0 ? kMaxPushSplits : kMaxSplits;
    if (splits > cap) splits = cap;
    // Short K (at most 64 chunks): the largest cluster whose clusters of all row tiles are
    // resident with one CTA per SM, launched with shared memory enough to keep two CTAs off an
    // SM, and with two converter groups and eight stages (six where eight do not fit) so that
    // the SM keeps as many converter warps and loads in flight as two CTAs would.  Fewer, longer splits on SMs of their own beat
    // two CTAs per SM here (the cluster's slowest CTA sets the reduction's end); long K keeps
    // the two-per-SM plan below.
    int one_sm = 0;
    if (p.KC <= 64) {
      constexpr size_t kOneSm = 116 * 1024;
      // every CTA needs a chunk of its own: at most KC splits
      for (int s = cap < p.KC ? cap : int(p.KC); s >= 2 && one_sm == 0; --s) {
        int st = 8;
        plan(s, st, &smem, &push, &rows_per, &rb_bytes);
        if (smem > size_t(227) * 1024) plan(s, st = 6, &smem, &push, &rows_per, &rb_bytes);
        if (!push && s > kMaxSplits) continue;
        const size_t sm = smem < kOneSm ? kOneSm : smem;
        if (sm > size_t(227) * 1024) continue;
        auto qk = st == 8 ? act_quant_kernel<true, false, 8> : act_quant_kernel<true, false, 6>;
        if (set_smem(qk, st == 8 ? 4 : 6, sm) != cudaSuccess) break;
        cudaLaunchConfig_t q{};
        q.gridDim = dim3(unsigned(s), unsigned(ag.MT), 1);
        q.blockDim = dim3(threads1(st), 1, 1);
        q.dynamicSmemBytes = sm;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = unsigned(s);
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        q.attrs = at;
        q.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, qk, &q) == cudaSuccess && int64_t(clusters) >= ag.MT) {
          one_sm = s;
          min_smem = sm;
          stages = st;
        }
      }
    }
    if (one_sm > 0) splits = 1;  // skip the two-per-SM search
    for (; splits > 1; --splits) {
      plan(splits, 4, &smem, &push, &rows_per, &rb_bytes);
      if (!push && splits > kMaxSplits) continue;  // pulled partials: at most a portable cluster
      cudaError_t e = set_smem(act_quant_kernel<false>, 0, smem);
      if (e != cudaSuccess) {
        *why = "cudaFuncSetAttribute(shared memory size / carveout) failed";
        return e;
      }
      cudaLaunchConfig_t q{};
      q.gridDim = dim3(unsigned(splits), unsigned(ag.MT), 1);
      q.blockDim = dim3(threads1(4), 1, 1);
      q.dynamicSmemBytes = smem;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = unsigned(splits);
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      q.attrs = at;
      q.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, act_quant_kernel<false>, &q) == cudaSuccess &&
          int64_t(clusters) >= ag.MT)
        break;
    }
    if (one_sm > 0) splits = one_sm;
  }
  if (cached == 0) {
    std::lock_guard<std::mutex> lk(plan_mu);
    if (planned.size() > 4096) planned.clear();
    planned[key] = {splits, stages, min_smem};
  }
  plan(splits, stages, &smem, &push, &rows_per, &rb_bytes);
  if (smem < min_smem) smem = min_smem;
  p.splits = splits;
  p.push = push;
  p.rows_per = rows_per;
  p.rb_bytes = rb_bytes;
  auto kernel = stages == 8 ? (a.int4 ? act_quant_kernel<true, true, 8> : act_quant_kernel<true, false, 8>)
                : stages == 6 ? (a.int4 ? act_quant_kernel<true, true, 6> : act_quant_kernel<true, false, 6>)
                : a.int4      ? (lowrank ? act_quant_kernel<true, true> : act_quant_kernel<false, true>)
                              : (lowrank ? act_quant_kernel<true> : act_quant_kernel<false>);
  const int slot = stages == 4 ? (lowrank ? 1 : 0) + (a.int4 ? 2 : 0) : (stages == 8 ? 4 : 6) + (a.int4 ? 1 : 0);
  {
    cudaError_t e = set_smem(kernel, slot, smem);
    if (e != cudaSuccess) {
      *why = "cudaFuncSetAttribute(shared memory size / carveout) failed";
      return e;
    }
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(splits), unsigned(ag.MT), 1);
  cfg.blockDim = dim3(threads1(stages), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (lowrank && splits > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = unsigned(splits);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, map, p);
  if (e != cudaSuccess) *why = "launch of the activation kernel failed";
  return e;
}

}  // namespace svdq
