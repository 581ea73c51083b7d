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
// Design (sm_100a): persistent CTA pairs (clusters of 2, one CTA per SM) over
// 256 x 256 output tiles with the 2-SM MMA (cta_group::2, M = 256):
//   * CTA v of a pair owns A rows [128 v, 128 v + 128) and B rows (output
//     features) [128 v, 128 v + 128) of the tile, and holds the tile's rows
//     [128 v, 128 v + 128) x 256 columns of the accumulator in its tensor
//     memory.  Sharing B across the pair cuts the operand bytes every SM
//     streams per FLOP by 30 % against a 128 x 256 one-SM tile; the freed
//     shared memory buys a fifth pipeline stage.
//   * warp 20 of each CTA fills a 5-stage ring with tensor loads (one per
//     operand, 2 KB rows) of the pre-tiled, pre-swizzled operands: A 16 KB and
//     the B half 16 KB counted on the leader CTA's full barrier (armed by the
//     leader with both CTAs' bytes), A scales 2 KB and all 256 rows of B scales
//     4 KB counted on the CTA's own scale barrier.  After the K loop of a tile
//     the same ring carries the lr' and L2^T chunks.
//   * warps 16-19 of each CTA (one per tensor-memory lane quarter) move each
//     stage's block scales from shared memory into their CTA's tensor memory
//     with tcgen05.st, in the replicated layout the block-scaled MMA reads,
//     then arrive on the leader's full barrier.  Scale staging therefore
//     never occupies the tensor pipe, which issues nothing but MMAs.
//   * warp 21 of the leader issues 4 block-scaled MMAs per 256-wide k-tile,
//     then the bf16 MMAs of the fold, and commits every stage back to both
//     CTAs' empty barriers with a multicast commit.
//   * warps 0-15 of each CTA: epilogue, one output row x 64 columns per
//     thread (warp w: lane quarter w % 4, columns 64 (w / 4) .. +63): tensor
//     memory -> registers, release the accumulator to the leader, then alpha,
//     bias, GELU -> bf16 while the next tile's K loop runs.  Each warp writes
//     32 rows x 16 columns at a time into its own 1 KB shared-memory buffer,
//     and one lane hands the buffer to a TMA tensor store: Y leaves in whole
//     sectors through the bulk-copy engine, not as row-strided stores that
//     would contend with the operand feed.
//   * The QKV instance (kQkv) finishes a fused Q|K|V projection instead
//     (Diffusers/Nunchaku page, fused-QKV section: projection, Q/K norm and
//     rotary embedding in one operator): each row's bf16 outputs of a Q or K
//     head of 128 columns are RMS-normalized over the head (the two warps
//     holding its halves swap their sums of squares through shared memory
//     under an mbarrier), scaled by norm_q / norm_k, turned pair by pair by
//     the row's rotary angles, and rounded to bf16 once more.  V passes.
//   * Tensor memory (per CTA): accumulator columns [0, 256), scale factors of
//     stage s at 256 + 16 s (A) and 336 + 32 s (B).
//   * Every wait is bounded (status word + clean exit on timeout); the pair
//     meets at a cluster barrier before freeing tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>

#include "int4.h"
#include "kernels.h"
#include "ptx.cuh"

namespace svdq {

namespace {

using namespace ptx;

constexpr int kStages2 = 5;
constexpr int kEpiWarps = 16;    // warp w: lane quarter w % 4, accumulator columns 64 (w / 4) .. +63
constexpr int kThreads2 = 704;  // warps 0-15 epilogue, 16-19 scales, 20 producer, 21 MMA
constexpr int kScaleWarp0 = 16, kProducerWarp = 20, kMmaWarp = 21;
constexpr int kFullArrivals = 1 + 2 * 4;  // leader producer + the scale warps of both CTAs
constexpr uint32_t kHalf = 128;                          // rows per CTA of A and of B
constexpr uint32_t kOffA = 0;                            // 16 KB
constexpr uint32_t kOffB = kHalf * kRowBytes;            // 16 KB
constexpr uint32_t kOffSFA = 2 * kHalf * kRowBytes;      // 2 KB
constexpr uint32_t kOffSFB = kOffSFA + kSFATileBytes;    // 4 KB
constexpr uint32_t kStage2 = kOffSFB + kSFBTileBytes;    // 38912 bytes
constexpr uint32_t kFoldBytes = 2 * kHalf * kRowBytes;   // lr' 16 KB + L2^T half 16 KB
constexpr uint32_t kCtrl2 = 256;
constexpr uint32_t kBiasBytes = kEpiWarps * 64 * 2;  // per epilogue warp: its 64 bias values (bf16)
constexpr uint32_t kXchBytes = 8 * 2 * 64 * 4;  // QKV: [head warp pair][parity][2 halves x 32 rows] floats
constexpr uint32_t kNormBytes = kEpiWarps * 64 * 4;  // QKV: per epilogue warp, its 64 norm_q and 64 norm_k weights
// Output staging: each epilogue warp writes 32 rows x 16 columns of Y (1 KB,
// 32-byte swizzle) to shared memory and one TMA store moves them to Y, so the
// output leaves through the bulk-copy engine in whole sectors instead of 32
// row-strided stores per instruction.  Two buffers per warp (one in the QKV
// instance, whose exchange and weights take the room).
constexpr uint32_t kYRows = 32, kYCols = 16, kYBufBytes = kYRows * kYCols * 2;
// The epilogue instances of the kernel.
enum EpiKind : int {
  kEpiPlain = 0,  // Y = bf16(act(alpha acc + b))
  kEpiQkv = 1,    // fused Q | K | V: per-head RMSNorm of Q and K, rotary turn, V unchanged
  kEpiMlp = 2,    // fused MLP pair: the next layer's NVFP4 activations instead of Y
};
// MLP instance: per epilogue warp, its 64 columns of the next layer's 1/lambda (float) and a
// 1 KB staging buffer of 32 rows x 16 columns of x_hat (the A fragments of the down
// projection).  After the down projection the four staging buffers of a lane quarter's warps
// hold the 32 rows x 32 ranks of partial x_hat L1 the four warps sum.
constexpr uint32_t kInv2Bytes = kEpiWarps * 64 * 4;
constexpr uint32_t kStgBytes = kEpiWarps * 1024;
constexpr uint32_t kRedBytes = 0;
template <int kEpi>
struct EpiSmem {
  static constexpr bool kQkv = kEpi == kEpiQkv, kMlp = kEpi == kEpiMlp;
  static constexpr int kYBufs = kMlp ? 0 : kQkv ? 1 : 2;
  static constexpr uint32_t kXch = kStages2 * kStage2 + kCtrl2 + kBiasBytes;  // QKV only
  static constexpr uint32_t kNorm = kXch + (kQkv ? kXchBytes : 0);
  static constexpr uint32_t kY = (kNorm + (kQkv ? kNormBytes : 0) + 1023u) & ~1023u;
  static constexpr uint32_t kInv2 = kY + kEpiWarps * kYBufs * kYBufBytes;  // MLP only
  static constexpr uint32_t kStg = kInv2 + (kMlp ? kInv2Bytes : 0);
  static constexpr uint32_t kRed = kStg + (kMlp ? kStgBytes : 0);
  static constexpr uint32_t kEnd = kRed + (kMlp ? kRedBytes : 0);
};
static_assert(EpiSmem<kEpiPlain>::kEnd + 1024 <= 227 * 1024, "shared memory budget (plain)");
static_assert(kEpiWarps * 4 * kYBufBytes <= kStages2 * kStage2, "last-tile staging fits in the stage ring");
static_assert(EpiSmem<kEpiQkv>::kEnd + 1024 <= 227 * 1024, "shared memory budget (QKV)");
static_assert(EpiSmem<kEpiMlp>::kEnd + 1024 <= 227 * 1024, "shared memory budget (MLP)");
constexpr uint32_t kTmemCols2 = 512;
constexpr uint32_t kColSFA = 256, kColSFB = kColSFA + 16 * kStages2;
constexpr uint16_t kPairMask = 0x3;

static_assert(kStage2 % 1024 == 0, "stage must keep 1 KB alignment");
static_assert(kColSFB + kStages2 * 32 <= kTmemCols2, "tensor memory budget");

// Every pre-tiled operand is viewed by its tensor map as rows of 2 KB (256
// elements of 8 bytes), so a 16 KB tile is one load of 8 such rows.
constexpr uint32_t kMapRow = 2048;
constexpr int kRowsA = kHalf * kRowBytes / kMapRow;         // 8: 128 rows of A (or lr')
constexpr int kRowsBTile = kBTileBytes / kMapRow;           // 16: a whole 256-row tile
constexpr int kRowsSFA = kSFATileBytes / kMapRow;           // 1
constexpr int kRowsSFB = kSFBTileBytes / kMapRow;           // 2

struct alignas(64) GemmMaps {
  CUtensorMap y;    // Y bf16 [M, N], box = 32 rows x 16 columns, 32-byte swizzle
  CUtensorMap a;    // act codes, box = 128 rows of one tile (16 KB)
  CUtensorMap asf;  // act scales, box = one k-tile (2 KB)
  CUtensorMap lr;   // lr' tiles, box = 16 KB
  CUtensorMap b;    // weight codes, box = half a 256-row tile (16 KB)
  CUtensorMap bsf;  // weight scales, box = one k-tile of all 256 rows (4 KB)
  CUtensorMap l2;   // L2^T tiles, box = half a tile (16 KB)
};

struct GemmParams {
  const uint16_t* bias;  // padded to NT * 256, or null
  uint16_t* Y;
  uint32_t* status;
  int32_t M, N, MP, NT, KT, RJ, r_tot, epilogue;
  float alpha;
  uint64_t timeout_ns;
  // QKV instance only
  const uint16_t* norm_q;  // bf16 [128]
  const uint16_t* norm_k;  // bf16 [128]
  const float* rope;       // packed rotary table: [row tile][32 chunks][128 rows] x 16 bytes
  float eps;
  int32_t qkv_cols;  // N / 3
  // MLP instance only: fc2's activation buffer (codes, scales), 1/lambda2, L1_2^T chunks
  uint8_t* codes2;
  uint8_t* sf2;
  const float* inv_lam2;
  const uint8_t* l1t2;
  float* partial;     // [NT][MP * 256][r2] fp32
  int32_t KT2, rc16_2, r2;
  float g_a2, c_a2;
};

__device__ __forceinline__ float gelu_tanh(float x) {
  const float k0 = 0.7978845608028654f;  // sqrt(2 / pi)
  const float u = k0 * (x + 0.044715f * x * x * x);
  return 0.5f * x * (1.0f + tanh_approx(u));
}

// Tile t -> (row-tile pair mp, weight tile nt).  Tiles run in groups of
// kGroupMP row-tile pairs swept across all weight tiles, so the tiles in flight
// at any time touch at most kGroupMP pairs' activations and a few weight tiles:
// both stay in L2 even when the whole operands do not.
constexpr int kGroupMP = 8;
__device__ __forceinline__ void tile_coords(const GemmParams& p, int tile, int& mp, int& nt) {
  const int per_group = kGroupMP * p.NT;
  const int grp = tile / per_group, in = tile % per_group;
  const int gsize = (p.MP - grp * kGroupMP) < kGroupMP ? (p.MP - grp * kGroupMP) : kGroupMP;
  mp = grp * kGroupMP + in % gsize;
  nt = in / gsize;
}

// 32 accumulator columns of one row -> alpha, bias, act -> 16 words of bf16 pairs.
// `bias` points at the 16 bf16 pairs of these columns' bias in shared memory (or null).
template <bool kMayGelu = true>
__device__ __forceinline__ void finish_chunk(const GemmParams& p, const uint32_t* v, const uint32_t* bias,
                                             uint32_t* out) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t bw = bias ? bias[e] : 0u;
    const float b0 = bf16lo(bw), b1 = bf16hi(bw);
    float y0 = fmaf(p.alpha, __uint_as_float(v[2 * e]), b0);
    float y1 = fmaf(p.alpha, __uint_as_float(v[2 * e + 1]), b1);
    if (kMayGelu && p.epilogue == SVDQ_EPI_GELU_TANH) {
      y0 = gelu_tanh(y0);
      y1 = gelu_tanh(y1);
    }
    out[e] = f32x2_to_bf16x2(y0, y1);
  }
}

// 16 columns of this thread's row (8 words of bf16 pairs) -> buffer `slot` of
// the warp's staging area (row = lane, two 16-byte chunks swizzled by bit 2 of
// the row) -> one TMA store of the warp's 32 rows x 16 columns at (x, y).
// Lane 0 owns the warp's bulk groups; a buffer is rewritten only after its
// last store has read it (kBufs buffers normally, 4 on the CTA's last tile).
template <int kBufs>
__device__ __forceinline__ void store_y16(const CUtensorMap* map, uint8_t* buf, uint32_t buf_s, bool last, int lane,
                                          const uint32_t* w, int32_t x, int32_t y, int32_t M, uint32_t& slot) {
  if (y >= M) return;  // all 32 rows are padding (the same for the whole warp)
  if (lane == 0) {
    if (last)
      bulk_wait_read<3>();
    else
      bulk_wait_read<kBufs - 1>();
  }
  __syncwarp();
  uint8_t* b = buf + slot * kYBufBytes + uint32_t(lane) * 32u;
  const uint32_t sw = (uint32_t(lane) >> 2) & 1u;
  *reinterpret_cast<uint4*>(b + 16u * sw) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(b + 16u * (sw ^ 1u)) = make_uint4(w[4], w[5], w[6], w[7]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, buf_s + slot * kYBufBytes, x, y);
    bulk_commit();
  }
  const uint32_t n = last ? 4u : uint32_t(kBufs);
  slot = slot + 1 == n ? 0u : slot + 1;
}

// kRopeBatch chunks (2 pairs each) of one Q or K head row: the bf16 values in
// out[2 kRopeBatch] are RMS-normalized with `inv`, scaled by the weights (bf16
// pairs in wsm) and turned by the (cos, sin, cos, sin) chunks in t.
#ifndef SVDQ_ROPE_BATCH
#define SVDQ_ROPE_BATCH 4
#endif
constexpr int kRopeBatch = SVDQ_ROPE_BATCH;
__device__ __forceinline__ void norm_rope_chunks(uint32_t* out, float inv, const uint32_t* wsm, const float4* t) {
#pragma unroll
  for (int e2 = 0; e2 < kRopeBatch; ++e2) {
    const uint2 w = *reinterpret_cast<const uint2*>(wsm + 2 * e2);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t y = out[2 * e2 + j], ww = j ? w.y : w.x;
      const float c = j ? t[e2].z : t[e2].x, sn = j ? t[e2].w : t[e2].y;
      const float z0 = bf16lo(y) * inv * bf16lo(ww);
      const float z1 = bf16hi(y) * inv * bf16hi(ww);
      out[2 * e2 + j] = f32x2_to_bf16x2(z0 * c - z1 * sn, z1 * c + z0 * sn);
    }
  }
}

// Fused MLP pair, second step: lr'2 = bf16(sum_t partial[t] / alpha2), the weight tiles t of
// fc1 added in order (deterministic), into fc2's activation buffer.
__global__ void mlp_reduce_kernel(const float* __restrict__ partial, int32_t nt, int64_t rows, int32_t r2,
                                  float inv_alpha2, uint8_t* lr2, int32_t RJ2) {
  griddep_wait();  // the partials are the previous kernel's output
  const int groups = r2 / 4;
  const int64_t total = rows * groups;
  const size_t plane = size_t(rows) * size_t(r2);
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int64_t m = idx / groups;
    const int c = int(idx % groups) * 4;
    const float* src = partial + size_t(m) * r2 + c;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int t = 0;
    for (; t + 8 <= nt; t += 8) {
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = __ldg(reinterpret_cast<const float4*>(src + size_t(t + j) * plane));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        acc.x += v[j].x;
        acc.y += v[j].y;
        acc.z += v[j].z;
        acc.w += v[j].w;
      }
    }
    for (; t < nt; ++t) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src + size_t(t) * plane));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    uint2 w;
    w.x = f32x2_to_bf16x2(__fmul_rn(acc.x, inv_alpha2), __fmul_rn(acc.y, inv_alpha2));
    w.y = f32x2_to_bf16x2(__fmul_rn(acc.z, inv_alpha2), __fmul_rn(acc.w, inv_alpha2));
    uint8_t* tile = lr2 + (size_t(m / kBM) * RJ2 + size_t(c / kRChunk)) * kATileBytes;
    *reinterpret_cast<uint2*>(tile + sw128(uint32_t(m % kBM), uint32_t(c % kRChunk) * 2u)) = w;
  }
}

__global__ void rope_pack_kernel(const float4* rope, int64_t M, float4* packed, int64_t total) {
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = idx % kBM, c = (idx / kBM) % kRopeChunks, t = idx / (int64_t(kBM) * kRopeChunks);
    const int64_t row = t * kBM + i;
    packed[idx] = row < M ? rope[row * kRopeChunks + c] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int kEpi>
__global__ void __launch_bounds__(kThreads2, 1) gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
  constexpr bool kQkv = kEpi == kEpiQkv, kMlp = kEpi == kEpiMlp;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;

  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const uint32_t rank = cluster_ctarank();  // 0 = leader of the pair
  const bool leader = rank == 0;
  const int pair = int(blockIdx.x >> 1), npairs = int(gridDim.x >> 1);

  uint8_t* ctrl = smem + kStages2 * kStage2;
  const uint32_t ctrl_s = sbase + kStages2 * kStage2;
  const uint32_t FULL = ctrl_s, EMPTY = ctrl_s + 40u;
  const uint32_t ACCF = ctrl_s + 80u, ACCE = ctrl_s + 88u, DRAIN = ctrl_s + 96u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 104);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(ctrl + 108);
  const uint32_t SFULL = ctrl_s + 112u;  // 5 barriers: this CTA's scales of a stage have landed
  uint32_t* bias_s = reinterpret_cast<uint32_t*>(ctrl + kCtrl2);  // [warp][32 bf16 pairs]
  const uint32_t XCH = ctrl_s + 152u;  // QKV: 8 barriers, one per warp pair sharing a head
  using ES = EpiSmem<kEpi>;
  float* xch = reinterpret_cast<float*>(smem + ES::kXch);
  uint32_t* norm_s = reinterpret_cast<uint32_t*>(smem + ES::kNorm);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(FULL + 8u * s, kFullArrivals);  // leader: producer (+ both CTAs' A/B bytes) + 8 scale warps
      mbar_init(EMPTY + 8u * s, 1);             // both: one multicast commit per phase
      mbar_init(SFULL + 8u * s, 1);             // both: own producer (+ own scale bytes)
    }
    mbar_init(ACCF, 1);   // both: one multicast commit per tile
    mbar_init(ACCE, 2 * kEpiWarps);  // leader: one arrival per epilogue warp of both CTAs
    mbar_init(DRAIN, 1);
    if (kQkv)
      for (int h = 0; h < 8; ++h) mbar_init(XCH + 8u * h, 64);  // every thread of both warps
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(ctrl_s + 104u, kTmemCols2);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the activation buffer is the previous kernel's output, Y may be its input
  griddep_wait();
  griddep_launch_dependents();

  auto fail = [&](uint32_t code) {
    *abort_flag = 1u;
    atomicOr(p.status, code);
  };

  const int ntiles = p.MP * p.NT;
  const int nlr = (p.r_tot + kRChunk - 1) / kRChunk;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&maps.a);
      prefetch_tensormap(&maps.b);
      prefetch_tensormap(&maps.asf);
      prefetch_tensormap(&maps.bsf);
      uint32_t it = 0;
      bool stop = false;
      for (int tile = pair; tile < ntiles && !stop; tile += npairs) {
        int mp, nt;
        tile_coords(p, tile, mp, nt);
        const int mt = 2 * mp + int(rank);
        for (int kt = 0; kt < p.KT; ++kt) {
          const uint32_t s = it % kStages2, ph = (it / kStages2) & 1u;
          if (!mbar_wait(EMPTY + 8u * s, ph ^ 1u, abort_flag, p.timeout_ns)) {
            fail(0x10u);
            stop = true;
            break;
          }
          const uint32_t st = sbase + s * kStage2;
          const uint32_t bar = mapa(FULL + 8u * s, 0u);
          if (leader) mbar_expect_tx(FULL + 8u * s, 2u * kOffSFA);
          mbar_expect_tx(SFULL + 8u * s, kStage2 - kOffSFA);
          tma_load_2d_pair(st + kOffA, &maps.a, 0, (mt * p.KT + kt) * kRowsA, bar);
          tma_load_2d_pair(st + kOffB, &maps.b, 0, (nt * p.KT + kt) * kRowsBTile + int(rank) * kRowsA, bar);
          tma_load_2d(st + kOffSFA, &maps.asf, 0, (mt * p.KT + kt) * kRowsSFA, SFULL + 8u * s);
          tma_load_2d(st + kOffSFB, &maps.bsf, 0, (nt * p.KT + kt) * kRowsSFB, SFULL + 8u * s);
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
          const uint32_t bar = mapa(FULL + 8u * s, 0u);
          if (leader) mbar_expect_tx(FULL + 8u * s, 2u * kFoldBytes);
          mbar_arrive(SFULL + 8u * s);  // no scales in a fold stage: the scale warps only pass it on
          tma_load_2d_pair(st + kOffA, &maps.lr, 0, (mt * p.RJ + j) * kRowsA, bar);
          tma_load_2d_pair(st + kOffB, &maps.l2, 0, (nt * p.RJ + j) * kRowsBTile + int(rank) * kRowsA, bar);
          ++it;
        }
      }
      // every issued copy (of both CTAs) must land before the pair may exit
      for (uint32_t i = it > kStages2 ? it - kStages2 : 0; i < it; ++i) {
        mbar_wait(SFULL + 8u * (i % kStages2), (i / kStages2) & 1u, nullptr, p.timeout_ns);
        if (leader) mbar_wait_cluster(FULL + 8u * (i % kStages2), (i / kStages2) & 1u, nullptr, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------ MMA issue (leader)
    if (leader && lane == 0) {
      const uint32_t id_fp4 = idesc_nvfp4_m256(kBN), id_bf16 = idesc_bf16_m256(kBN);
      uint32_t it = 0, tc = 0;
      bool stop = false, any = false;
      for (int tile = pair; tile < ntiles && !stop; tile += npairs) {
        if (!mbar_wait(ACCE, (tc & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
          fail(0x20u);
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < p.KT; ++kt) {
          const uint32_t s = it % kStages2, ph = (it / kStages2) & 1u;
          if (!mbar_wait_cluster(FULL + 8u * s, ph, abort_flag, p.timeout_ns)) {
            fail(0x20u);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * kStage2;
          const uint32_t sfa = tmem + kColSFA + 16u * s, sfb = tmem + kColSFB + 32u * s;
#pragma unroll
          for (uint32_t kb = 0; kb < 4; ++kb)
            umma_nvfp4_pair(tmem, sdesc_sw128(st + kOffA + 32u * kb), sdesc_sw128(st + kOffB + 32u * kb), id_fp4,
                            sfa + 4u * kb, sfb + 8u * kb, (kt | int(kb)) ? 1u : 0u);
          tc_commit_pair_mc(EMPTY + 8u * s, kPairMask);
          any = true;
          ++it;
        }
        for (int j = 0; j < nlr && !stop; ++j) {
          const uint32_t s = it % kStages2, ph = (it / kStages2) & 1u;
          if (!mbar_wait_cluster(FULL + 8u * s, ph, abort_flag, p.timeout_ns)) {
            fail(0x20u);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * kStage2;
          const int left = p.r_tot - kRChunk * j;
          const int nks = (left < kRChunk ? left : kRChunk) / 16;
          for (int ks = 0; ks < nks; ++ks)
            umma_bf16_pair(tmem, sdesc_sw128(st + kOffA + 32u * ks), sdesc_sw128(st + kOffB + 32u * ks), id_bf16, 1u);
          tc_commit_pair_mc(EMPTY + 8u * s, kPairMask);
          ++it;
        }
        if (stop) break;
        tc_commit_pair_mc(ACCF, kPairMask);
        ++tc;
      }
      if (any) {
        tc_commit_pair(DRAIN);
        mbar_wait(DRAIN, 0u, nullptr, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp >= kScaleWarp0) {  // warps 16-19
    // --------------------------------------------------------- scale warps
    // Warp w writes tensor-memory lanes 32 q .. 32 q + 31, q = w % 4.  For k block
    // kb the MMA reads A scales at column 256 + 16 s + 4 kb and B scales at
    // 336 + 32 s + 8 kb (B rows 0-127) and + 4 (rows 128-255), with lane i of
    // every quarter holding word w = row i + 32 w of each 512-byte atom: the
    // atom's 16-byte row i replicated into every quarter.
    const uint32_t q = uint32_t(warp & 3);
    const uint32_t lanes = (32u * q) << 16;
    uint32_t it = 0;
    bool stop = false;
    for (int tile = pair; tile < ntiles && !stop; tile += npairs) {
      for (int k = 0; k < p.KT + nlr && !stop; ++k) {
        const uint32_t s = it % kStages2, ph = (it / kStages2) & 1u;
        bool ok = mbar_wait(SFULL + 8u * s, ph, abort_flag, p.timeout_ns);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0 && *abort_flag == 0u) fail(0x80u);
          stop = true;
          break;
        }
        if (k < p.KT) {
          const uint8_t* st = smem + s * kStage2;
          {
            uint32_t r[16];
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint4 a = *reinterpret_cast<const uint4*>(st + kOffSFA + kb * kSFAtomBytes + lane * 16);
              r[4 * kb] = a.x, r[4 * kb + 1] = a.y, r[4 * kb + 2] = a.z, r[4 * kb + 3] = a.w;
            }
            tmem_st16(tmem + lanes + kColSFA + 16u * s, r);
          }
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t r[16];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const uint4 b = *reinterpret_cast<const uint4*>(st + kOffSFB + (4 * half + h) * kSFAtomBytes + lane * 16);
              r[4 * h] = b.x, r[4 * h + 1] = b.y, r[4 * h + 2] = b.z, r[4 * h + 3] = b.w;
            }
            tmem_st16(tmem + lanes + kColSFB + 32u * s + 16u * half, r);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(FULL + 8u * s, 0u);
        ++it;
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    // warp w reads TMEM lanes 32 (w % 4) .. +31 and accumulator columns
    // 64 (w / 4) .. +63: its share of the tile goes to registers, the
    // accumulator is released to the leader, then the rows are finished and
    // stored while the next tile's K loop runs.
    uint32_t tc = 0, xc = 0, yslot = 0;
    const int quarter = warp & 3, colq = warp >> 2;
    uint8_t* ybuf = smem + ES::kY + uint32_t(warp) * ES::kYBufs * kYBufBytes;
    const uint32_t ybuf_s = sbase + ES::kY + uint32_t(warp) * ES::kYBufs * kYBufBytes;
    uint32_t* norm_w = norm_s + warp * 64;  // QKV: [Q, K][32 bf16 pairs] of this warp's columns
    float* inv2_w = reinterpret_cast<float*>(smem + ES::kInv2) + warp * 64;  // MLP: 1/lambda2 of its columns
    if (kQkv) {
      const int half = colq & 1;
      norm_w[lane] = *reinterpret_cast<const uint32_t*>(p.norm_q + half * 64 + 2 * lane);
      norm_w[32 + lane] = *reinterpret_cast<const uint32_t*>(p.norm_k + half * 64 + 2 * lane);
      __syncwarp();
    }
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t tl = tmem + (uint32_t(quarter * 32) << 16) + uint32_t(colq * 64);
    for (int tile = pair; tile < ntiles; tile += npairs) {
      int mp, nt;
      tile_coords(p, tile, mp, nt);
      const int mt = 2 * mp + int(rank);
      // stage this warp's 64 bias values (warp-private; the previous tile's reads are done)
      uint32_t* bias_w = bias_s + warp * 32;
      __syncwarp();
      if (p.bias) bias_w[lane] = *reinterpret_cast<const uint32_t*>(p.bias + size_t(nt) * kBN + colq * 64 + lane * 2);
      if constexpr (kMlp) {  // and its 64 values of the next layer's 1/lambda (its input channels)
        const int n0s = nt * kBN + colq * 64;
        if (n0s < p.N) {
          const float2 w2 = *reinterpret_cast<const float2*>(p.inv_lam2 + n0s + 2 * lane);
          inv2_w[2 * lane] = w2.x;
          inv2_w[2 * lane + 1] = w2.y;
        }
      }
      __syncwarp();
      bool ok = mbar_wait(ACCF, tc & 1u, abort_flag, p.timeout_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (*abort_flag == 0u) fail(0x40u);
        break;
      }
      tc_fence_after();
      uint32_t v[64];
      tmem_ld32(tl, v);
      tmem_ld32(tl + 32u, v + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(ACCE, 0u);  // this warp's share of the accumulator is free
      const int32_t y0 = mt * kBM + quarter * 32;  // first row of this warp's share
      // On its last tile the CTA's stage ring is idle (every MMA that read it
      // has completed): each warp stages its 4 stores there, 4 KB apart, and
      // never waits for a buffer.
      const bool last = tile + npairs >= ntiles;
      if (last) yslot = 0;
      uint8_t* const sbuf = last ? smem + uint32_t(warp) * 4u * kYBufBytes : ybuf;
      const uint32_t sbuf_s = last ? sbase + uint32_t(warp) * 4u * kYBufBytes : ybuf_s;
      auto put16 = [&](const uint32_t* w, int32_t x) {
        store_y16<ES::kYBufs>(&maps.y, sbuf, sbuf_s, last, lane, w, x, y0, p.M, yslot);
      };
      if constexpr (kQkv) {
        // the two warps of a head (colq 2h, 2h + 1) agree on every branch
        // below: the head's columns are all below N or all above (N % 128 == 0)
        const int n0 = nt * kBN + colq * 64;
        if (n0 < p.N) {
          uint32_t out[32];
          finish_chunk<false>(p, v, p.bias ? bias_w : nullptr, out);
          finish_chunk<false>(p, v + 32, p.bias ? bias_w + 16 : nullptr, out + 16);
          const int part = n0 / p.qkv_cols;  // 0 Q, 1 K, 2 V
          if (part < 2) {
            float ss = 0.0f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              uint32_t o = out[e];
              asm volatile("" : "+r"(o));  // keep the packed words, not their unpacked floats, across the wait
              const float y0 = bf16lo(o), y1 = bf16hi(o);
              ss = fmaf(y0, y0, ss);
              ss = fmaf(y1, y1, ss);
            }
            const int hp = quarter + 4 * (colq >> 1), half = colq & 1;
            // this row's (cos, sin) chunks: coalesced across the warp's rows;
            // the first batch is in flight while the two warps meet
            const float4* cs = reinterpret_cast<const float4*>(p.rope) +
                               (size_t(mt) * kRopeChunks + size_t(half) * 16) * kBM + size_t(row_in_tile);
            float4 t[kRopeBatch];
#pragma unroll
            for (int j = 0; j < kRopeBatch; ++j) t[j] = __ldg(cs + j * kBM);
            float* xb = xch + (hp * 2 + int(xc & 1u)) * 64;
            xb[half * 32 + lane] = ss;
            mbar_arrive(XCH + 8u * hp);
            bool okx = mbar_wait(XCH + 8u * hp, xc & 1u, abort_flag, p.timeout_ns);
            okx = __all_sync(0xFFFFFFFFu, okx);
            if (!okx) {
              if (*abort_flag == 0u) fail(0x80u);
              break;
            }
            ++xc;
            const float tot = xb[lane] + xb[32 + lane];  // the same order in both warps
            const float inv = rsqrtf(fmaf(tot, 1.0f / 128.0f, p.eps));
            const uint32_t* wsm = norm_w + part * 32;
#pragma unroll
            for (int b = 0; b < 16 / kRopeBatch; ++b) {
              if (b) {
#pragma unroll
                for (int j = 0; j < kRopeBatch; ++j) t[j] = __ldg(cs + (b * kRopeBatch + j) * kBM);
              }
              norm_rope_chunks(out + 2 * kRopeBatch * b, inv, wsm + 2 * kRopeBatch * b, t);
            }
          }
          // rows past M are clipped by the tensor store
#pragma unroll
          for (int j = 0; j < 4; ++j) put16(out + 8 * j, n0 + 16 * j);
        }
      } else if constexpr (kMlp) {
        // the next layer's (fc2's) activations from this row's 64 outputs: x_hat2 =
        // bf16(y / lambda2), NVFP4 codes and block scales into fc2's activation buffer (fc1's
        // weight tile nt is fc2's k-tile nt, this warp's 64 columns its chunk colq), then the
        // partial x_hat2 L1_2 over these 64 inputs on the warp-level tensor cores
        const int n0 = nt * kBN + colq * 64;
        const bool in = n0 < p.N;  // warp-uniform: N % 64 == 0
        uint32_t xh[32];
        uint32_t cw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}, sc4 = 0u;
        if (in) {
          uint32_t y[32];
          finish_chunk(p, v, p.bias ? bias_w : nullptr, y);
          finish_chunk(p, v + 32, p.bias ? bias_w + 16 : nullptr, y + 16);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            float xf[16];
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float lo = __fmul_rn(bf16lo(y[8 * b + j]), inv2_w[16 * b + 2 * j]);
              const float hi = __fmul_rn(bf16hi(y[8 * b + j]), inv2_w[16 * b + 2 * j + 1]);
              const uint32_t h = f32x2_to_bf16x2(lo, hi);
              xh[8 * b + j] = h;
              xf[2 * j] = bf16lo(h);
              xf[2 * j + 1] = bf16hi(h);
              amax = fmaxf(amax, fmaxf(fabsf(xf[2 * j]), fabsf(xf[2 * j + 1])));
            }
            const uint32_t sc = f32_to_e4m3(__fmul_rn(amax, p.c_a2));
            const float d = __fmul_rn(e4m3_value(sc), p.g_a2);
            const float rcp = d == 0.0f ? 0.0f : __frcp_rn(d);
            cw[2 * b] = f32x8_to_e2m1(__fmul_rn(xf[0], rcp), __fmul_rn(xf[1], rcp), __fmul_rn(xf[2], rcp),
                                      __fmul_rn(xf[3], rcp), __fmul_rn(xf[4], rcp), __fmul_rn(xf[5], rcp),
                                      __fmul_rn(xf[6], rcp), __fmul_rn(xf[7], rcp));
            cw[2 * b + 1] = f32x8_to_e2m1(__fmul_rn(xf[8], rcp), __fmul_rn(xf[9], rcp), __fmul_rn(xf[10], rcp),
                                          __fmul_rn(xf[11], rcp), __fmul_rn(xf[12], rcp), __fmul_rn(xf[13], rcp),
                                          __fmul_rn(xf[14], rcp), __fmul_rn(xf[15], rcp));
            sc4 |= sc << (8 * b);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) xh[j] = 0u;
        }
        {  // columns past N (fc2's K) get zero codes and scales, like padding read past the end of X
          uint8_t* ctile = p.codes2 + (size_t(mt) * p.KT2 + nt) * kATileBytes;
          *reinterpret_cast<uint4*>(ctile + sw128(uint32_t(row_in_tile), uint32_t(colq) * 32u)) =
              make_uint4(cw[0], cw[1], cw[2], cw[3]);
          *reinterpret_cast<uint4*>(ctile + sw128(uint32_t(row_in_tile), uint32_t(colq) * 32u + 16u)) =
              make_uint4(cw[4], cw[5], cw[6], cw[7]);
          uint8_t* stile = p.sf2 + (size_t(mt) * p.KT2 + nt) * kSFATileBytes + size_t(colq) * kSFAtomBytes;
          *reinterpret_cast<uint32_t*>(stile + sf_atom(uint32_t(row_in_tile), 0u)) = sc4;
        }
        // partial x_hat2 L1_2, up to 32 ranks at a time: the warp's 32 rows x 16 inputs of x_hat2
        // go through its staging buffer (row = lane, 16-byte halves swizzled by bit 2 of the
        // row) into A fragments; L1_2^T words straight from global memory are the B fragments
        uint8_t* stg = smem + ES::kStg + uint32_t(warp) * 1024u;
        const uint32_t stg_s = sbase + ES::kStg + uint32_t(warp) * 1024u;
        // the reduction slot of fragment value f (0..31) of this lane: the staging buffer of the
        // quarter's warp quarter + 4 (f / 8), float (f % 8) * 32 + lane
        auto red_slot = [&](int f) {
          return reinterpret_cast<float*>(smem + ES::kStg + uint32_t(quarter + 4 * (f >> 3)) * 1024u) +
                 (f & 7) * 32 + lane;
        };
        const uint8_t* l1c = p.l1t2 + size_t(in ? n0 / 64 : 0) * size_t(p.rc16_2) * 128u;
        const uint32_t swz = (uint32_t(lane) >> 2) & 1u;
        for (int rc = 0; rc < p.r2; rc += 32) {
          const int nb8 = p.r2 - rc >= 32 ? 4 : 2;  // ranks come in multiples of 16
          float acc[2][4][4];
#pragma unroll
          for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[a][b][e] = 0.0f;
          if (in) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              uint32_t bf[4][2];
#pragma unroll
              for (int n8 = 0; n8 < 4; ++n8) {  // B fragments first: their loads overlap the staging
                const uint32_t rho = uint32_t(rc + 8 * n8 + (lane >> 2));
                const uint32_t kb = uint32_t(32 * kk + 4 * (lane & 3));
                bf[n8][0] = n8 < nb8 ? __ldg(reinterpret_cast<const unsigned int*>(l1c + sw128(rho, kb))) : 0u;
                bf[n8][1] = n8 < nb8 ? __ldg(reinterpret_cast<const unsigned int*>(l1c + sw128(rho, kb + 16u))) : 0u;
              }
              *reinterpret_cast<uint4*>(stg + lane * 32 + 16u * swz) =
                  make_uint4(xh[8 * kk], xh[8 * kk + 1], xh[8 * kk + 2], xh[8 * kk + 3]);
              *reinterpret_cast<uint4*>(stg + lane * 32 + 16u * (swz ^ 1u)) =
                  make_uint4(xh[8 * kk + 4], xh[8 * kk + 5], xh[8 * kk + 6], xh[8 * kk + 7]);
              __syncwarp();
              uint32_t af[2][4];
#pragma unroll
              for (int m16 = 0; m16 < 2; ++m16) {
                const uint32_t row = uint32_t(m16 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8);
                const uint32_t kh = uint32_t(lane >> 4);
                ldsm_x4(stg_s + row * 32u + ((kh ^ ((row >> 2) & 1u)) * 16u), af[m16]);
              }
              __syncwarp();
#pragma unroll
              for (int n8 = 0; n8 < 4; ++n8)
                if (n8 < nb8) {
                  mma_bf16_16816(acc[0][n8], af[0], bf[n8][0], bf[n8][1]);
                  mma_bf16_16816(acc[1][n8], af[1], bf[n8][0], bf[n8][1]);
                }
            }
          }
          // the quarter's four warps add their partials in column order (deterministic), the
          // last one writes the tile's partial of these 32 rows x nb8 * 8 ranks; the staging
          // buffers become the sum's storage once all four warps are past their MMAs
          const uint32_t bar = 1u + uint32_t(quarter);
          named_sync(bar, 128);
#pragma unroll
          for (int step = 0; step < 4; ++step) {
            if (colq == step) {
#pragma unroll
              for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b)
                  if (b < nb8) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                      float* slot = red_slot((a * 4 + b) * 4 + e);
                      if (step) acc[a][b][e] += *slot;
                      if (step < 3) *slot = acc[a][b][e];
                    }
                  }
              if (step == 3) {
                const int64_t rows = int64_t(p.MP) * 2 * kBM;
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                  for (int b = 0; b < 4; ++b)
                    if (b < nb8) {
#pragma unroll
                      for (int hh = 0; hh < 2; ++hh) {
                        const int64_t r = int64_t(mt) * kBM + quarter * 32 + a * 16 + (lane >> 2) + 8 * hh;
                        const int rk = rc + 8 * b + 2 * (lane & 3);
                        *reinterpret_cast<float2*>(p.partial + (size_t(nt) * rows + r) * p.r2 + rk) =
                            make_float2(acc[a][b][2 * hh], acc[a][b][2 * hh + 1]);
                      }
                    }
              }
            }
            named_sync(bar, 128);
          }
        }
      } else {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int n0 = nt * kBN + colq * 64 + q * 32;
          if (n0 < p.N) {  // N % 64 == 0: the warp's 64 columns are all in or all out
            uint32_t out[16];
            finish_chunk(p, v + 32 * q, p.bias ? bias_w + q * 16 : nullptr, out);
            put16(out, n0);
            put16(out + 8, n0 + 16);
          }
        }
      }
      ++tc;
    }
    if (lane == 0) bulk_wait_read<0>();  // the staging buffers are read before the CTA may exit
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  cluster_sync();  // both CTAs are done with every MMA, copy and tensor-memory read
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols2);
  }
}

// ------------------------------------------------------------------ INT4 layer
// Kernel 2 of the INT4 layer (int4.h): the same persistent CTA pairs, tile
// order, fold of the low-rank branch and plain epilogue as gemm_kernel; the
// mainloop differs.  tcgen05 has no 4-bit integer MMA kind, so per group of
// 64 inputs:
//   * the producer (warp 24) copies this CTA's raw INT4 blocks of A (128 rows)
//     and B (its 128 of the tile's 256 rows) and their bf16 scales (8.5 KB);
//   * two groups of widening warps (16-19 and 20-23) take alternate groups of
//     64, so two are widened at once.  Thread t widens row t of A and of B to
//     f16 values q s 2^e (q s is exact in f16 for a bf16 s, and the prescale
//     2^e keeps it inside f16's range): the row of A into tensor memory
//     (tcgen05.st, the warp's own lane quarter), the row of B into the
//     128-byte-swizzled K-major tile in shared memory;
//   * the leader (warp 25) issues 4 MMAs of kind::f16 (M = 256, N = 256,
//     K = 16), A from tensor memory and B from shared memory.
// A in tensor memory keeps 32 KB per stage (the widened A written and read
// back) off shared memory.  Inside a group of 8 inputs the widened values sit
// in the order 0 4 1 5 2 6 3 7 (two nibbles per 32-bit lane of the
// unpacking); A and B share that order, so the sum over K is unchanged.
constexpr int kStages4 = 4;
constexpr int kConvWarp0 = 16;  // warps 16-23 widen the codes, in two groups of 4
constexpr uint32_t kOffA4 = 0;                           // the fold's lr' chunk (16 KB)
constexpr uint32_t kOffB4 = kHalf * kRowBytes;           // f16 B: this CTA's 128 rows x 64 (16 KB)
constexpr uint32_t kOffRawA4 = 2 * kHalf * kRowBytes;    // INT4 block of A (4 KB)
constexpr uint32_t kOffRawB4 = kOffRawA4 + kBlock4Bytes;  // INT4 block of B (4 KB)
constexpr uint32_t kOffSA4 = kOffRawB4 + kBlock4Bytes;   // 128 bf16 scales of A
constexpr uint32_t kOffSB4 = kOffSA4 + kScale4Bytes;     // 128 bf16 scales of B
constexpr uint32_t kRaw4Bytes = 2 * kBlock4Bytes + 2 * kScale4Bytes;
constexpr uint32_t kStage4 = (kOffSB4 + kScale4Bytes + 1023u) & ~1023u;  // 41 KB
constexpr int kFullArrivals4 = 1 + 2 * 4;  // leader producer + one widening group of both CTAs
constexpr int kThreads4 = 832, kProducerWarp4 = 24, kMmaWarp4 = 25;  // 16 epilogue + 8 widening + 2
constexpr uint32_t kTmemCols4 = 512;  // accumulator 256 + A of 4 stages x 32
constexpr uint32_t kColA4 = 256;
constexpr uint32_t kY4 = (kStages4 * kStage4 + kCtrl2 + kBiasBytes + 1023u) & ~1023u;
constexpr uint32_t kEnd4 = kY4 + kEpiWarps * 2 * kYBufBytes;
static_assert(kStage4 % 1024 == 0, "stage must keep 1 KB alignment");
static_assert(kEnd4 + 1024 <= 227 * 1024, "shared memory budget (INT4)");
static_assert(kEpiWarps * 4 * kYBufBytes <= kStages4 * kStage4, "last-tile staging fits in the stage ring");

struct Int4Params {
  const uint8_t* a_codes;  // activation INT4 blocks [MT][KC][4 KB]
  const uint8_t* a_sf;     // activation scales [MT][KC][128] bf16
  const uint8_t* b_codes;  // weight INT4 blocks [NT][KC][2][4 KB]
  const uint8_t* b_sf;     // weight scales [NT][KC][256] bf16
  const uint16_t* bias;    // padded to NT * 256, or null
  uint16_t* Y;
  uint32_t* status;
  int32_t M, N, MP, NT, KC, KG, RJ, r_tot, epilogue;
  float alpha, pre_a, pre_w;
  uint64_t timeout_ns;
};

__host__ __device__ constexpr uint32_t idesc_f16_m256(int n) {
  return (1u << 4)                    // D format: f32; A, B: f16 (format fields 0)
         | (uint32_t(n >> 3) << 17)   // N / 8
         | (uint32_t(256 >> 4) << 24);
}

// Row t of a 128-row INT4 block and its bf16 scale -> 64 f16 values q s pre,
// written as row t of a 128-byte-swizzled K-major tile.  The scale saturates
// at 9352, the largest f16 value whose sevenfold stays finite in f16 (7 x 9352
// rounds to 65472): a clamp at 65504 / 7 itself would round up to 9360 in f16,
// and 7 x 9360 = 65520 rounds to infinity.  So no value overflows.
constexpr float kMaxWideScale4 = 9352.0f;  // largest f16 s with 7 s finite in f16
__device__ __forceinline__ void widen_int4_row(const uint8_t* raw, const uint8_t* sc, float pre, uint8_t* dst,
                                               uint32_t t) {
  const uint4 c0 = *reinterpret_cast<const uint4*>(raw + t * 16u);          // inputs 0..31
  const uint4 c1 = *reinterpret_cast<const uint4*>(raw + 2048u + t * 16u);  // inputs 32..63
  const uint32_t sb = *reinterpret_cast<const uint16_t*>(sc + t * 2u);
  const float s = fminf(__uint_as_float(sb << 16) * pre, kMaxWideScale4);
  uint32_t s2;
  asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(s2) : "f"(s));
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  // nibble u (two's complement q) -> f16 1024 + (u ^ 8) = 1032 + q: one LOP3 per two values;
  // subtracting 1032 leaves q exactly
  constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x64086408u;  // kMagic as f16x2 is (1032, 1032)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w = words[i];
    uint32_t v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t h = kMagic ^ ((w >> (4 * j)) & kMask);  // inputs 8 i + j (low), 8 i + j + 4 (high)
      uint32_t q;
      asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(h), "r"(kMagic));
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(v[j]) : "r"(q), "r"(s2));
    }
    *reinterpret_cast<uint4*>(dst + sw128(t, 16u * uint32_t(i))) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

// The same widening into 32 registers (64 f16 values of row t, pairs in the smem order) for a
// tensor-memory store: register 4 i + j holds inputs 8 i + j (low) and 8 i + j + 4 (high).
__device__ __forceinline__ void widen_int4_row_regs(const uint8_t* raw, const uint8_t* sc, float pre, uint32_t t,
                                                    uint32_t* out) {
  const uint4 c0 = *reinterpret_cast<const uint4*>(raw + t * 16u);
  const uint4 c1 = *reinterpret_cast<const uint4*>(raw + 2048u + t * 16u);
  const uint32_t sb = *reinterpret_cast<const uint16_t*>(sc + t * 2u);
  const float s = fminf(__uint_as_float(sb << 16) * pre, kMaxWideScale4);
  uint32_t s2;
  asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(s2) : "f"(s));
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x64086408u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w = words[i];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t h = kMagic ^ ((w >> (4 * j)) & kMask);
      uint32_t q;
      asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(h), "r"(kMagic));
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[4 * i + j]) : "r"(q), "r"(s2));
    }
  }
}

// D (+)= A(tensor memory) B(shared memory)^T, both CTAs of the pair, kind::f16.
__device__ __forceinline__ void umma_f16_tmem_a_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(kThreads4, 1) gemm_int4_kernel(const __grid_constant__ GemmMaps maps,
                                                                 const Int4Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;

  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const uint32_t rank = cluster_ctarank();  // 0 = leader of the pair
  const bool leader = rank == 0;
  const int pair = int(blockIdx.x >> 1), npairs = int(gridDim.x >> 1);

  uint8_t* ctrl = smem + kStages4 * kStage4;
  const uint32_t ctrl_s = sbase + kStages4 * kStage4;
  const uint32_t FULL = ctrl_s, EMPTY = ctrl_s + 32u, RAW = ctrl_s + 64u;
  const uint32_t ACCF = ctrl_s + 96u, ACCE = ctrl_s + 104u, DRAIN = ctrl_s + 112u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 120);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(ctrl + 124);
  uint32_t* bias_s = reinterpret_cast<uint32_t*>(ctrl + kCtrl2);  // [warp][32 bf16 pairs]

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages4; ++s) {
      mbar_init(FULL + 8u * s, kFullArrivals4);  // leader: producer (+ fold bytes) + 8 widening warps
      mbar_init(EMPTY + 8u * s, 1);              // both: one multicast commit per phase
      mbar_init(RAW + 8u * s, 1);                // both: own producer (+ own raw bytes)
    }
    mbar_init(ACCF, 1);
    mbar_init(ACCE, 2 * kEpiWarps);
    mbar_init(DRAIN, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp4) {
    tmem_alloc_pair(ctrl_s + 120u, kTmemCols4);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  griddep_launch_dependents();

  auto fail = [&](uint32_t code) {
    *abort_flag = 1u;
    atomicOr(p.status, code);
  };

  const int ntiles = p.MP * p.NT;
  const int nlr = (p.r_tot + kRChunk - 1) / kRChunk;
  const int tiles_mp = p.MP, tiles_nt = p.NT;
  auto coords = [&](int tile, int& mp, int& nt) {
    const int per_group = kGroupMP * tiles_nt;
    const int grp = tile / per_group, in = tile % per_group;
    const int gsize = (tiles_mp - grp * kGroupMP) < kGroupMP ? (tiles_mp - grp * kGroupMP) : kGroupMP;
    mp = grp * kGroupMP + in % gsize;
    nt = in / gsize;
  };

  if (warp == kProducerWarp4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&maps.lr);
      prefetch_tensormap(&maps.l2);
      uint32_t it = 0;
      bool stop = false;
      for (int tile = pair; tile < ntiles && !stop; tile += npairs) {
        int mp, nt;
        coords(tile, mp, nt);
        const int mt = 2 * mp + int(rank);
        for (int c = 0; c < p.KG; ++c) {
          const uint32_t s = it % kStages4, ph = (it / kStages4) & 1u;
          if (!mbar_wait(EMPTY + 8u * s, ph ^ 1u, abort_flag, p.timeout_ns)) {
            fail(0x10u);
            stop = true;
            break;
          }
          const uint32_t st = sbase + s * kStage4;
          if (leader) mbar_arrive(FULL + 8u * s);  // no bytes: the widening warps fill the operands
          mbar_expect_tx(RAW + 8u * s, kRaw4Bytes);
          const size_t ablk = size_t(mt) * p.KC + size_t(c);
          const size_t bblk = size_t(nt) * p.KC + size_t(c);
          bulk_g2s(st + kOffRawA4, p.a_codes + ablk * kBlock4Bytes, kBlock4Bytes, RAW + 8u * s);
          bulk_g2s(st + kOffSA4, p.a_sf + ablk * kScale4Bytes, kScale4Bytes, RAW + 8u * s);
          bulk_g2s(st + kOffRawB4, p.b_codes + (bblk * 2 + rank) * kBlock4Bytes, kBlock4Bytes, RAW + 8u * s);
          bulk_g2s(st + kOffSB4, p.b_sf + (bblk * 2 + rank) * kScale4Bytes, kScale4Bytes, RAW + 8u * s);
          ++it;
        }
        for (int j = 0; j < nlr && !stop; ++j) {
          const uint32_t s = it % kStages4, ph = (it / kStages4) & 1u;
          if (!mbar_wait(EMPTY + 8u * s, ph ^ 1u, abort_flag, p.timeout_ns)) {
            fail(0x10u);
            stop = true;
            break;
          }
          const uint32_t st = sbase + s * kStage4;
          const uint32_t bar = mapa(FULL + 8u * s, 0u);
          if (leader) mbar_expect_tx(FULL + 8u * s, 2u * kFoldBytes);
          mbar_arrive(RAW + 8u * s);  // nothing to widen: the warps only pass the stage on
          tma_load_2d_pair(st + kOffA4, &maps.lr, 0, (mt * p.RJ + j) * kRowsA, bar);
          tma_load_2d_pair(st + kOffB4, &maps.l2, 0, (nt * p.RJ + j) * kRowsBTile + int(rank) * kRowsA, bar);
          ++it;
        }
      }
      // every issued copy (of both CTAs) must land before the pair may exit
      for (uint32_t i = it > kStages4 ? it - kStages4 : 0; i < it; ++i) {
        mbar_wait(RAW + 8u * (i % kStages4), (i / kStages4) & 1u, nullptr, p.timeout_ns);
        if (leader) mbar_wait_cluster(FULL + 8u * (i % kStages4), (i / kStages4) & 1u, nullptr, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp4) {
    // ------------------------------------------------------ MMA issue (leader)
    if (leader && lane == 0) {
      const uint32_t id_f16 = idesc_f16_m256(kBN), id_bf16 = idesc_bf16_m256(kBN);
      uint32_t it = 0, tc = 0;
      bool stop = false, any = false;
      for (int tile = pair; tile < ntiles && !stop; tile += npairs) {
        if (!mbar_wait(ACCE, (tc & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
          fail(0x20u);
          break;
        }
        tc_fence_after();
        for (int c = 0; c < p.KG; ++c) {
          const uint32_t s = it % kStages4, ph = (it / kStages4) & 1u;
          if (!mbar_wait_cluster(FULL + 8u * s, ph, abort_flag, p.timeout_ns)) {
            fail(0x20u);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * kStage4;
#pragma unroll
          for (uint32_t kk = 0; kk < 4; ++kk)
            umma_f16_tmem_a_pair(tmem, tmem + kColA4 + 32u * s + 8u * kk, sdesc_sw128(st + kOffB4 + 32u * kk), id_f16,
                                 (c | int(kk)) ? 1u : 0u);
          tc_commit_pair_mc(EMPTY + 8u * s, kPairMask);
          any = true;
          ++it;
        }
        for (int j = 0; j < nlr && !stop; ++j) {
          const uint32_t s = it % kStages4, ph = (it / kStages4) & 1u;
          if (!mbar_wait_cluster(FULL + 8u * s, ph, abort_flag, p.timeout_ns)) {
            fail(0x20u);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * kStage4;
          const int left = p.r_tot - kRChunk * j;
          const int nks = (left < kRChunk ? left : kRChunk) / 16;
          for (int ks = 0; ks < nks; ++ks)
            umma_bf16_pair(tmem, sdesc_sw128(st + kOffA4 + 32u * ks), sdesc_sw128(st + kOffB4 + 32u * ks), id_bf16,
                           1u);
          tc_commit_pair_mc(EMPTY + 8u * s, kPairMask);
          ++it;
        }
        if (stop) break;
        tc_commit_pair_mc(ACCF, kPairMask);
        ++tc;
      }
      if (any) {
        tc_commit_pair(DRAIN);
        mbar_wait(DRAIN, 0u, nullptr, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp >= kConvWarp0) {  // warps 16-23
    // ---------------------------------------------------- widening warps
    const uint32_t t = uint32_t((warp - kConvWarp0) & 3) * 32u + uint32_t(lane);  // row of A and of B
    const uint32_t lanes = (uint32_t((warp - kConvWarp0) & 3) * 32u) << 16;  // this warp's lane quarter
    const uint32_t grp = uint32_t(warp - kConvWarp0) >> 2;  // group 0 takes the even stages, group 1 the odd
    uint32_t it = 0;
    bool stop = false;
    for (int tile = pair; tile < ntiles && !stop; tile += npairs) {
      for (int k = 0; k < p.KG + nlr && !stop; ++k) {
        const uint32_t s = it % kStages4, ph = (it / kStages4) & 1u;
        if ((it & 1u) != grp) {
          ++it;
          continue;
        }
        bool ok = mbar_wait(RAW + 8u * s, ph, abort_flag, p.timeout_ns);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0 && *abort_flag == 0u) fail(0x80u);
          stop = true;
          break;
        }
        if (k < p.KG) {
          uint8_t* st = smem + s * kStage4;
          {
            uint32_t a[32];
            widen_int4_row_regs(st + kOffRawA4, st + kOffSA4, p.pre_a, t, a);
            tmem_st32(tmem + lanes + kColA4 + 32u * s, a);
          }
          widen_int4_row(st + kOffRawB4, st + kOffSB4, p.pre_w, st + kOffB4, t);
          tmem_wait_st();
          fence_proxy_async_smem();  // generic writes -> tensor-core reads
          tc_fence_before();
        }
        __syncwarp();
        // the peer's warps arrive remotely at CTA scope, as the NVFP4 scale warps do (an arrive
        // with release at cluster scope costs about 900 clocks on the stage's critical path)
        if (lane == 0) {
          if (leader)
            mbar_arrive(FULL + 8u * s);
          else
            mbar_arrive_cluster(FULL + 8u * s, 0u);
        }
        ++it;
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    // as the plain instance of gemm_kernel: warp w reads TMEM lanes 32 (w % 4)
    // .. +31 and accumulator columns 64 (w / 4) .. +63, releases the
    // accumulator, then alpha, bias, GELU -> bf16 -> TMA tensor stores
    uint32_t tc = 0, yslot = 0;
    const int quarter = warp & 3, colq = warp >> 2;
    uint8_t* ybuf = smem + kY4 + uint32_t(warp) * 2u * kYBufBytes;
    const uint32_t ybuf_s = sbase + kY4 + uint32_t(warp) * 2u * kYBufBytes;
    const uint32_t tl = tmem + (uint32_t(quarter * 32) << 16) + uint32_t(colq * 64);
    for (int tile = pair; tile < ntiles; tile += npairs) {
      int mp, nt;
      coords(tile, mp, nt);
      const int mt = 2 * mp + int(rank);
      uint32_t* bias_w = bias_s + warp * 32;
      __syncwarp();
      if (p.bias) bias_w[lane] = *reinterpret_cast<const uint32_t*>(p.bias + size_t(nt) * kBN + colq * 64 + lane * 2);
      __syncwarp();
      bool ok = mbar_wait(ACCF, tc & 1u, abort_flag, p.timeout_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (*abort_flag == 0u) fail(0x40u);
        break;
      }
      tc_fence_after();
      uint32_t v[64];
      tmem_ld32(tl, v);
      tmem_ld32(tl + 32u, v + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(ACCE, 0u);  // this warp's share of the accumulator is free
      const int32_t y0 = mt * kBM + quarter * 32;
      const bool last = tile + npairs >= ntiles;
      if (last) yslot = 0;
      uint8_t* const sbuf = last ? smem + uint32_t(warp) * 4u * kYBufBytes : ybuf;
      const uint32_t sbuf_s = last ? sbase + uint32_t(warp) * 4u * kYBufBytes : ybuf_s;
      GemmParams fp{};  // the fields finish_chunk reads
      fp.alpha = p.alpha;
      fp.epilogue = p.epilogue;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int n0 = nt * kBN + colq * 64 + q * 32;
        if (n0 < p.N) {
          uint32_t out[16];
          finish_chunk(fp, v + 32 * q, p.bias ? bias_w + q * 16 : nullptr, out);
          store_y16<2>(&maps.y, sbuf, sbuf_s, last, lane, out, n0, y0, p.M, yslot);
          store_y16<2>(&maps.y, sbuf, sbuf_s, last, lane, out + 8, n0 + 16, y0, p.M, yslot);
        }
      }
      ++tc;
    }
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  cluster_sync();  // both CTAs are done with every MMA, copy and tensor-memory read
  if (warp == kMmaWarp4) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols4);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// A pre-tiled operand of `bytes` bytes viewed as rows of 2 KB; one load = `box` rows.
bool encode_rows(CUtensorMap* m, const void* base, uint64_t bytes, uint32_t box) {
  auto enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {kMapRow / 8u, bytes / kMapRow};
  const cuuint64_t strides[1] = {kMapRow};
  const cuuint32_t boxd[2] = {kMapRow / 8u, box};
  const cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void*>(base), dims, strides, boxd, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Y bf16 [M, N] row-major for the epilogue's tensor stores: box 32 rows x 16 columns.
bool encode_y(CUtensorMap* m, void* Y, int64_t M, int64_t N) {
  auto enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cuuint64_t(N), cuuint64_t(M)};
  const cuuint64_t strides[1] = {cuuint64_t(N) * 2u};
  const cuuint32_t boxd[2] = {kYCols, kYRows};
  const cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, dims, strides, boxd, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm(const GemmLaunch& a, cudaStream_t s, const char** why) {
  const LayerGeom& lg = a.lg;
  const ActGeom ag = make_act_geom(lg, a.M);
  GemmMaps maps;
  const uint8_t* act = a.act;
  const uint8_t* lay = a.layer;
  const bool mlp = a.mlp_act2 != nullptr;
  bool ok = encode_rows(&maps.a, act + ag.off_codes, uint64_t(ag.MT) * ag.KT * kATileBytes, kRowsA) &&
            encode_rows(&maps.asf, act + ag.off_sf, uint64_t(ag.MT) * ag.KT * kSFATileBytes, kRowsSFA) &&
            encode_rows(&maps.b, lay + lg.off_bcodes, uint64_t(lg.NT) * lg.KT * kBTileBytes, kRowsA) &&
            encode_rows(&maps.bsf, lay + lg.off_sfb, uint64_t(lg.NT) * lg.KT * kSFBTileBytes, kRowsSFB) &&
            (mlp || encode_y(&maps.y, a.Y, a.M, lg.N));
  if (mlp) maps.y = maps.a;  // the MLP instance writes no Y
  if (ok && lg.RJ > 0) {
    ok = encode_rows(&maps.lr, act + ag.off_lr, uint64_t(ag.MT) * ag.RJ * kATileBytes, kRowsA) &&
         encode_rows(&maps.l2, lay + lg.off_l2t, uint64_t(lg.NT) * lg.RJ * kBTileBytes, kRowsA);
  } else {
    maps.lr = maps.a;  // never read without low-rank chunks
    maps.l2 = maps.b;
  }
  if (!ok) {
    *why = "cuTensorMapEncodeTiled rejected a GEMM operand";
    return cudaErrorInvalidValue;
  }
  GemmParams p{};
  p.bias = a.has_bias ? reinterpret_cast<const uint16_t*>(lay + lg.off_bias) : nullptr;
  p.Y = static_cast<uint16_t*>(a.Y);
  p.status = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(lay) + lg.off_status);
  p.M = int32_t(a.M);
  p.N = int32_t(lg.N);
  p.MP = int32_t(ag.MT / 2);
  p.NT = int32_t(lg.NT);
  p.KT = int32_t(lg.KT);
  p.RJ = int32_t(lg.RJ);
  p.r_tot = a.r_tot;
  p.epilogue = a.epilogue;
  p.alpha = a.alpha;
  p.timeout_ns = a.timeout_ns;
  const bool qkv = a.qkv_cols > 0;
  p.norm_q = a.norm_q;
  p.norm_k = a.norm_k;
  p.rope = a.rope;
  p.eps = a.eps;
  p.qkv_cols = a.qkv_cols;
  if (mlp) {
    const LayerGeom& g2 = a.mlp_lg2;
    const ActGeom ag2 = make_act_geom(g2, a.M);
    p.codes2 = a.mlp_act2 + ag2.off_codes;
    p.sf2 = a.mlp_act2 + ag2.off_sf;
    p.inv_lam2 = reinterpret_cast<const float*>(a.mlp_layer2 + g2.off_inv_lam);
    p.l1t2 = a.mlp_layer2 + g2.off_l1t;
    p.partial = a.mlp_partial;
    p.KT2 = int32_t(g2.KT);
    p.rc16_2 = int32_t(g2.RC16);
    p.r2 = a.mlp_r2;
    p.g_a2 = a.mlp_g_a2;
    p.c_a2 = a.mlp_c_a2;
  }
  const int kind = qkv ? kEpiQkv : mlp ? kEpiMlp : kEpiPlain;
  auto kernel = qkv ? gemm_kernel<kEpiQkv> : mlp ? gemm_kernel<kEpiMlp> : gemm_kernel<kEpiPlain>;

  const int64_t ntiles = int64_t(p.MP) * lg.NT;
  if (ntiles > (int64_t(1) << 30)) {
    *why = "problem too large for one launch";
    return cudaErrorInvalidValue;
  }
  const size_t smem = size_t(qkv   ? EpiSmem<kEpiQkv>::kEnd
                             : mlp ? EpiSmem<kEpiMlp>::kEnd
                                   : EpiSmem<kEpiPlain>::kEnd) +
                      1024;
  static std::atomic<int> max_pairs_of[3][64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::atomic<int>* max_pairs = max_pairs_of[kind];
  if (max_pairs[dev & 63].load() == 0) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               int(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) {
      *why = "cudaFuncSetAttribute(shared memory size / carveout) failed";
      return e;
    }
    cudaLaunchConfig_t q{};
    q.gridDim = dim3(2 * unsigned(a.num_sms / 2), 1, 1);
    q.blockDim = dim3(kThreads2, 1, 1);
    q.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    q.attrs = at;
    q.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kernel, &q);
    if (e != cudaSuccess || clusters < 1) {
      *why = "no CTA pair of the GEMM fits on this device";
      return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
    }
    max_pairs[dev & 63].store(clusters);
  }
  const int cap = max_pairs[dev & 63].load();
  const int pairs = int(ntiles < cap ? ntiles : cap);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreads2, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, maps, p);
  if (e != cudaSuccess) *why = "launch of the GEMM kernel failed";
  return e;
}

cudaError_t launch_gemm_int4(const Int4GemmLaunch& a, cudaStream_t s, const char** why) {
  const LayerGeom& lg = a.lg;
  const ActGeom ag = make_act_geom(lg, a.M);
  GemmMaps maps;
  const uint8_t* act = a.act;
  const uint8_t* lay = a.layer;
  bool ok = encode_y(&maps.y, a.Y, a.M, lg.N);
  if (ok && lg.RJ > 0) {
    ok = encode_rows(&maps.lr, act + ag.off_lr, uint64_t(ag.MT) * ag.RJ * kATileBytes, kRowsA) &&
         encode_rows(&maps.l2, lay + lg.off_l2t, uint64_t(lg.NT) * lg.RJ * kBTileBytes, kRowsA);
  } else {
    maps.lr = maps.y;  // never read without low-rank chunks
    maps.l2 = maps.y;
  }
  maps.a = maps.asf = maps.b = maps.bsf = maps.y;  // the INT4 operands arrive by bulk copies
  if (!ok) {
    *why = "cuTensorMapEncodeTiled rejected a GEMM operand";
    return cudaErrorInvalidValue;
  }
  Int4Params p{};
  p.a_codes = act + ag.off_codes;
  p.a_sf = act + ag.off_sf;
  p.b_codes = lay + lg.off_bcodes;
  p.b_sf = lay + lg.off_sfb;
  p.bias = a.has_bias ? reinterpret_cast<const uint16_t*>(lay + lg.off_bias) : nullptr;
  p.Y = static_cast<uint16_t*>(a.Y);
  p.status = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(lay) + lg.off_status);
  p.M = int32_t(a.M);
  p.N = int32_t(lg.N);
  p.MP = int32_t(ag.MT / 2);
  p.NT = int32_t(lg.NT);
  p.KC = int32_t(lg.KC);
  p.KG = int32_t(lg.K / kGroup4);
  p.RJ = int32_t(lg.RJ);
  p.r_tot = a.r_tot;
  p.epilogue = a.epilogue;
  p.alpha = a.alpha;
  p.pre_a = a.pre_a;
  p.pre_w = a.pre_w;
  p.timeout_ns = a.timeout_ns;
  const int64_t ntiles = int64_t(p.MP) * lg.NT;
  if (ntiles > (int64_t(1) << 30)) {
    *why = "problem too large for one launch";
    return cudaErrorInvalidValue;
  }
  const size_t smem = size_t(kEnd4) + 1024;
  static std::atomic<int> max_pairs[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (max_pairs[dev & 63].load() == 0) {
    cudaError_t e = cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               int(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) {
      *why = "cudaFuncSetAttribute(shared memory size / carveout) failed";
      return e;
    }
    cudaLaunchConfig_t q{};
    q.gridDim = dim3(2 * unsigned(a.num_sms / 2), 1, 1);
    q.blockDim = dim3(kThreads4, 1, 1);
    q.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    q.attrs = at;
    q.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, gemm_int4_kernel, &q);
    if (e != cudaSuccess || clusters < 1) {
      *why = "no CTA pair of the INT4 GEMM fits on this device";
      return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
    }
    max_pairs[dev & 63].store(clusters);
  }
  const int cap = max_pairs[dev & 63].load();
  const int pairs = int(ntiles < cap ? ntiles : cap);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreads4, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_int4_kernel, maps, p);
  if (e != cudaSuccess) *why = "launch of the INT4 GEMM kernel failed";
  return e;
}

size_t mlp_partial_bytes(int64_t NT1, int64_t MT, int32_t r2) {
  return size_t(NT1) * size_t(MT) * kBM * size_t(r2) * sizeof(float);
}

cudaError_t launch_mlp_reduce(const MlpReduceLaunch& a, cudaStream_t s) {
  const int64_t total = a.rows * (a.r2 / 4);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 8192) blocks = 8192;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mlp_reduce_kernel, a.partial, a.nt, a.rows, a.r2, a.inv_alpha2, a.lr2, a.RJ2);
}

cudaError_t launch_rope_pack(const float* rope, int64_t M, float* packed, cudaStream_t s) {
  const int64_t total = int64_t(rope_packed_bytes(M) / 16);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  rope_pack_kernel<<<unsigned(blocks), 256, 0, s>>>(reinterpret_cast<const float4*>(rope), M,
                                                    reinterpret_cast<float4*>(packed), total);
  return cudaGetLastError();
}

}  // namespace svdq
