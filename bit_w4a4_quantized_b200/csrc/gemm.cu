// gemm.cu -- kernel 2: W4A4 NVFP4 GEMM with the low-rank up projection folded into the
// same tensor-memory accumulator, and a bias (+ tanh-GELU) bf16 epilogue.
//
// SVDQuant summary page: section 3 (XW ~ s_X s_W Q_X Q_W: scales factor out of
// the low-bit product), section 4.2 (XW = X_hat L1 L2 + X_hat R, the 16-bit
// branch plus the 4-bit residual) and section 4.3 "Nunchaku" (Figure 6(b)):
// the up projection is fused into the 4-bit GEMM so the branch adds no pass
// over Y.  Here:
//   acc  = sum_k (e2m1(a) sa)(e2m1(w) sw)        tcgen05.mma kind::mxf4nvf4, block16
//   acc += lr' L2                                 tcgen05.mma kind::f16, same TMEM tile
//   Y    = bf16(act(alpha * acc + b)),  alpha = g_a g_w,  lr' = (X_hat L1) / alpha
//
// Design (sm_100a), persistent, one CTA per SM, 128 x 256 output tiles:
//   * warp 8: one thread fills a 4-stage ring with 1D bulk copies (every
//     operand is stored pre-tiled and pre-swizzled, so a stage is 4 copies:
//     A codes 16 KB, B codes 32 KB, A scales 2 KB, B scales 4 KB); after the K
//     loop of a tile it loads the lr' and L2^T chunks into the same ring;
//   * warp 9: one thread copies the stage's block scales into tensor memory
//     (tcgen05.cp 32x128b.warpx4), issues 4 block-scaled MMAs per 256-wide
//     k-tile, then the bf16 MMAs of the fold, and commits stages back;
//   * warps 0-7: epilogue, one output row x 128 columns per thread: tensor
//     memory -> registers, release the accumulator, then alpha, bias, GELU ->
//     bf16 -> global while the next tile's K loop runs.
//   * Tensor memory: accumulator columns [0, 256), scale factors of stage s at
//     256 + 16 s (A) and 320 + 32 s (B).
//   * Every wait is bounded (status word + clean exit on timeout).
#include <cuda_runtime.h>

#include <atomic>

#include "kernels.h"
#include "ptx.cuh"

namespace svdq {

namespace {

using namespace ptx;

constexpr int kStages2 = 4;
constexpr int kThreads2 = 320;  // warps 0-7 epilogue, 8 producer, 9 MMA
constexpr int kEpiThreads = 256;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr uint32_t kOffA = 0, kOffB = kATileBytes, kOffSFA = kOffB + kBTileBytes;
constexpr uint32_t kOffSFB = kOffSFA + kSFATileBytes;
constexpr uint32_t kStage2 = kOffSFB + kSFBTileBytes;  // 55296 bytes
constexpr uint32_t kCtrl2 = 128;
constexpr uint32_t kBiasBytes = 8 * 2 * 128 * 4;  // per epilogue warp: 2 tiles x 128 floats
constexpr uint32_t kTmemCols2 = 512;
constexpr uint32_t kColSFA = 256, kColSFB = 320;

static_assert(kStage2 % 1024 == 0, "stage must keep 1 KB alignment");
static_assert(kColSFB + kStages2 * 32 <= kTmemCols2, "tensor memory budget");

struct GemmParams {
  const uint8_t* a_codes;
  const uint8_t* a_sf;
  const uint8_t* a_lr;
  const uint8_t* b_codes;
  const uint8_t* b_sf;
  const uint8_t* b_l2t;
  const uint16_t* bias;  // padded to NT * 256, or null
  uint16_t* Y;
  uint32_t* status;
  int32_t M, N, MT, NT, KT, RJ, r_tot, epilogue;
  float alpha;
  uint64_t timeout_ns;
};

__device__ __forceinline__ float gelu_tanh(float x) {
  const float k0 = 0.7978845608028654f;  // sqrt(2 / pi)
  const float u = k0 * (x + 0.044715f * x * x * x);
  return 0.5f * x * (1.0f + tanh_approx(u));
}

// 32 accumulator columns of one row -> alpha, bias, act -> bf16 -> 64 bytes of Y.
// `bias` points at the 32 bias values of these columns in shared memory (or null).
__device__ __forceinline__ void store_chunk(const GemmParams& p, const uint32_t* v, const float* bias, int64_t row,
                                            int n0) {
  uint32_t out[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float b0 = bias ? bias[2 * e] : 0.0f, b1 = bias ? bias[2 * e + 1] : 0.0f;
    float y0 = fmaf(p.alpha, __uint_as_float(v[2 * e]), b0);
    float y1 = fmaf(p.alpha, __uint_as_float(v[2 * e + 1]), b1);
    if (p.epilogue == SVDQ_EPI_GELU_TANH) {
      y0 = gelu_tanh(y0);
      y1 = gelu_tanh(y1);
    }
    out[e] = f32x2_to_bf16x2(y0, y1);
  }
  uint4* dst = reinterpret_cast<uint4*>(p.Y + row * p.N + n0);
#pragma unroll
  for (int q = 0; q < 4; ++q) dst[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
}

__global__ void __launch_bounds__(kThreads2, 1) gemm_kernel(const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;

  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  uint8_t* ctrl = smem + kStages2 * kStage2;
  const uint32_t ctrl_s = sbase + kStages2 * kStage2;
  const uint32_t FULL = ctrl_s, EMPTY = ctrl_s + 32u;
  const uint32_t ACCF = ctrl_s + 64u, ACCE = ctrl_s + 72u, DRAIN = ctrl_s + 80u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 88);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(ctrl + 92);
  float* bias_s = reinterpret_cast<float*>(ctrl + kCtrl2);  // [warp][tile parity][128] floats

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(FULL + 8u * s, 1);
      mbar_init(EMPTY + 8u * s, 1);
    }
    mbar_init(ACCF, 1);
    mbar_init(ACCE, kEpiThreads);
    mbar_init(DRAIN, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(ctrl_s + 88u, kTmemCols2);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](uint32_t code) {
    *abort_flag = 1u;
    atomicOr(p.status, code);
  };

  const int ntiles = p.MT * p.NT;
  const int nlr = (p.r_tot + kRChunk - 1) / kRChunk;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool stop = false;
      for (int tile = int(blockIdx.x); tile < ntiles && !stop; tile += int(gridDim.x)) {
        const int mt = tile % p.MT, nt = tile / p.MT;
        for (int kt = 0; kt < p.KT; ++kt) {
          const uint32_t s = it % kStages2, ph = (it / kStages2) & 1u;
          if (!mbar_wait(EMPTY + 8u * s, ph ^ 1u, abort_flag, p.timeout_ns)) {
            fail(0x10u);
            stop = true;
            break;
          }
          const uint32_t st = sbase + s * kStage2;
          const uint32_t bar = FULL + 8u * s;
          mbar_expect_tx(bar, kStage2);
          bulk_g2s(st + kOffA, p.a_codes + (size_t(mt) * p.KT + kt) * kATileBytes, kATileBytes, bar);
          bulk_g2s(st + kOffB, p.b_codes + (size_t(nt) * p.KT + kt) * kBTileBytes, kBTileBytes, bar);
          bulk_g2s(st + kOffSFA, p.a_sf + (size_t(mt) * p.KT + kt) * kSFATileBytes, kSFATileBytes, bar);
          bulk_g2s(st + kOffSFB, p.b_sf + (size_t(nt) * p.KT + kt) * kSFBTileBytes, kSFBTileBytes, bar);
          ++it;
        }
        for (int j = 0; j < nlr && !stop; ++j) {
          const uint32_t s = it % kStages2, ph = (it / kStages2) & 1u;
          if (!mbar_wait(EMPTY + 8u * s, ph ^ 1u, abort_flag, p.timeout_ns)) {
            fail(0x10u);
            stop = true;
            break;
          }
          const uint32_t st = sbase + s * kStage2;
          const uint32_t bar = FULL + 8u * s;
          mbar_expect_tx(bar, kATileBytes + kBTileBytes);
          bulk_g2s(st + kOffA, p.a_lr + (size_t(mt) * p.RJ + j) * kATileBytes, kATileBytes, bar);
          bulk_g2s(st + kOffB, p.b_l2t + (size_t(nt) * p.RJ + j) * kBTileBytes, kBTileBytes, bar);
          ++it;
        }
      }
      // every issued copy must land before this CTA may exit
      for (uint32_t i = it > kStages2 ? it - kStages2 : 0; i < it; ++i)
        mbar_wait(FULL + 8u * (i % kStages2), (i / kStages2) & 1u, nullptr, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t id_fp4 = idesc_nvfp4(kBN), id_bf16 = idesc_bf16(kBN);
      uint32_t it = 0, tc = 0;
      bool stop = false, any = false;
      for (int tile = int(blockIdx.x); tile < ntiles && !stop; tile += int(gridDim.x)) {
        if (!mbar_wait(ACCE, (tc & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
          fail(0x20u);
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < p.KT; ++kt) {
          const uint32_t s = it % kStages2, ph = (it / kStages2) & 1u;
          if (!mbar_wait(FULL + 8u * s, ph, abort_flag, p.timeout_ns)) {
            fail(0x20u);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * kStage2;
          const uint32_t sfa = tmem + kColSFA + 16u * s, sfb = tmem + kColSFB + 32u * s;
#pragma unroll
          for (uint32_t kb = 0; kb < 4; ++kb) {
            tc_cp_32x128b_warpx4(sfa + 4u * kb, sdesc_sf(st + kOffSFA + kb * kSFAtomBytes));
            tc_cp_32x128b_warpx4(sfb + 8u * kb, sdesc_sf(st + kOffSFB + (2u * kb) * kSFAtomBytes));
            tc_cp_32x128b_warpx4(sfb + 8u * kb + 4u, sdesc_sf(st + kOffSFB + (2u * kb + 1u) * kSFAtomBytes));
          }
#pragma unroll
          for (uint32_t kb = 0; kb < 4; ++kb)
            umma_nvfp4(tmem, sdesc_sw128(st + kOffA + 32u * kb), sdesc_sw128(st + kOffB + 32u * kb), id_fp4,
                       sfa + 4u * kb, sfb + 8u * kb, (kt | int(kb)) ? 1u : 0u);
          tc_commit(EMPTY + 8u * s);
          any = true;
          ++it;
        }
        for (int j = 0; j < nlr && !stop; ++j) {
          const uint32_t s = it % kStages2, ph = (it / kStages2) & 1u;
          if (!mbar_wait(FULL + 8u * s, ph, abort_flag, p.timeout_ns)) {
            fail(0x20u);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * kStage2;
          const int left = p.r_tot - kRChunk * j;
          const int nks = (left < kRChunk ? left : kRChunk) / 16;
          for (int ks = 0; ks < nks; ++ks)
            umma_bf16(tmem, sdesc_sw128(st + kOffA + 32u * ks), sdesc_sw128(st + kOffB + 32u * ks), id_bf16, 1u);
          tc_commit(EMPTY + 8u * s);
          ++it;
        }
        if (stop) break;
        tc_commit(ACCF);
        ++tc;
      }
      if (any) {
        tc_commit(DRAIN);
        mbar_wait(DRAIN, 0u, nullptr, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue
    // warp w reads TMEM lanes 32 (w % 4) .. +31 (its lane quarter) and
    // accumulator columns 128 (w / 4) .. +127: the whole 128 x 256 tile is
    // read into registers, the accumulator is released, then the rows are
    // finished and stored while the next tile's K loop runs.
    uint32_t tc = 0;
    const int quarter = warp & 3, colhalf = warp >> 2;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t tl = tmem + (uint32_t(quarter * 32) << 16) + uint32_t(colhalf * 128);
    for (int tile = int(blockIdx.x); tile < ntiles; tile += int(gridDim.x)) {
      const int mt = tile % p.MT, nt = tile / p.MT;
      // stage this warp's 128 bias values while the K loop runs (warp-private,
      // double buffered by tile parity: only __syncwarp is needed)
      float* bias_w = bias_s + (size_t(warp) * 2 + (tc & 1u)) * 128;
      if (p.bias) {
        const uint2 w = *reinterpret_cast<const uint2*>(p.bias + size_t(nt) * kBN + colhalf * 128 + lane * 4);
        *reinterpret_cast<float4*>(bias_w + lane * 4) = make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
      }
      __syncwarp();
      bool ok = mbar_wait(ACCF, tc & 1u, abort_flag, p.timeout_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (*abort_flag == 0u) fail(0x40u);
        break;
      }
      tc_fence_after();
      uint32_t v[128];
      tmem_ld32(tl, v);
      tmem_ld32(tl + 32u, v + 32);
      tmem_ld32(tl + 64u, v + 64);
      tmem_ld32(tl + 96u, v + 96);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(ACCE);  // the accumulator may be overwritten now
      const int64_t row = int64_t(mt) * kBM + row_in_tile;
      if (row < p.M) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c0 = colhalf * 128 + q * 32;
          const int n0 = nt * kBN + c0;
          if (n0 < p.N) store_chunk(p, v + 32 * q, p.bias ? bias_w + q * 32 : nullptr, row, n0);
        }
      }
      ++tc;
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols2);
  }
}

}  // namespace

cudaError_t launch_gemm(const GemmLaunch& a, cudaStream_t s, const char** why) {
  const LayerGeom& lg = a.lg;
  const ActGeom ag = make_act_geom(lg, a.M);
  GemmParams p{};
  p.a_codes = a.act + ag.off_codes;
  p.a_sf = a.act + ag.off_sf;
  p.a_lr = a.act + ag.off_lr;
  p.b_codes = a.layer + lg.off_bcodes;
  p.b_sf = a.layer + lg.off_sfb;
  p.b_l2t = a.layer + lg.off_l2t;
  p.bias = a.has_bias ? reinterpret_cast<const uint16_t*>(a.layer + lg.off_bias) : nullptr;
  p.Y = static_cast<uint16_t*>(a.Y);
  p.status = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.layer) + lg.off_status);
  p.M = int32_t(a.M);
  p.N = int32_t(lg.N);
  p.MT = int32_t(ag.MT);
  p.NT = int32_t(lg.NT);
  p.KT = int32_t(lg.KT);
  p.RJ = int32_t(lg.RJ);
  p.r_tot = a.r_tot;
  p.epilogue = a.epilogue;
  p.alpha = a.alpha;
  p.timeout_ns = a.timeout_ns;

  const int64_t ntiles = ag.MT * lg.NT;
  if (ntiles > (int64_t(1) << 30)) {
    *why = "too many output tiles";
    return cudaErrorInvalidValue;
  }
  const size_t smem = size_t(kStages2) * kStage2 + kCtrl2 + kBiasBytes + 1024;
  {
    static std::atomic<int> set_on[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (!set_on[dev & 63].load()) {
      cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      if (e != cudaSuccess) {
        *why = "cudaFuncSetAttribute(max dynamic shared memory) failed";
        return e;
      }
      set_on[dev & 63].store(1);
    }
  }
  const int grid = int(ntiles < a.num_sms ? ntiles : a.num_sms);
  gemm_kernel<<<grid, kThreads2, smem, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) *why = "launch of the GEMM kernel failed";
  return e;
}

}  // namespace svdq
