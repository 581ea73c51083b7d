// lora.cu -- attach / detach a LoRA adapter on the low-rank branch, and the
// bounded-wait test kernel.
//
// Abstract of arXiv 2411.05007 (SVDQuant): the engine supports off-the-shelf
// LoRAs without re-quantization.  With smoothing, X A B = X_hat (diag(lambda) A) B,
// so the adapter joins the branch as extra ranks
//   L1' = [L1 | bf16(lambda A scale)],  L2' = [L2 ; B]
// and R (the 4-bit residual) is untouched.  This kernel rewrites ranks
// [rank, rank_capacity) of the tiled L1^T and L2^T operands; ranks beyond the
// adapter are zeroed.
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace svdq {

namespace {

__global__ void lora_swap_kernel(uint8_t* layer, LayerGeom g, const uint16_t* A, const uint16_t* B, int r_e,
                                 float scale) {
  const int64_t r0 = g.rank;
  const int64_t nr = int64_t(g.rcap) - r0;
  const int64_t kc = g.KC * kKChunk;  // padded K
  const int64_t nn = g.NT * kBN;      // padded N
  const int64_t total1 = nr * kc, total2 = nr * nn;
  const float* lam = reinterpret_cast<const float*>(layer + g.off_lam);
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total1 + total2;
       idx += int64_t(gridDim.x) * blockDim.x) {
    if (idx < total1) {
      const int64_t i = idx / kc, k = idx % kc;  // adapter rank i, input feature k
      uint16_t v = 0;
      if (i < r_e && k < g.K) {
        const float a = __uint_as_float(uint32_t(A[k * r_e + i]) << 16);
        const float s = __fmul_rn(__fmul_rn(lam[k], a), scale);
        v = uint16_t(ptx::f32x2_to_bf16x2(s, 0.0f) & 0xFFFFu);
      }
      *reinterpret_cast<uint16_t*>(layer + l1t_off(g, r0 + i, k)) = v;
    } else {
      const int64_t j = idx - total1;
      const int64_t i = j % nr, n = j / nr;  // adapter rank i, output feature n
      uint16_t v = 0;
      if (i < r_e && n < g.N) v = B[i * g.N + n];
      *reinterpret_cast<uint16_t*>(layer + l2t_off(g, n, r0 + i)) = v;
    }
  }
}

__device__ uint32_t g_bounded_wait_status;

__global__ void bounded_wait_test_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&bar), 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the wait must give up by itself
    const bool ok = ptx::mbar_wait(ptx::smem_u32(&bar), 0u, &abort_flag, timeout_ns);
    g_bounded_wait_status = ok ? 0u : 1u;
  }
}

}  // namespace

cudaError_t launch_lora_swap(const LoraLaunch& a, cudaStream_t s) {
  const int64_t nr = int64_t(a.lg.rcap) - a.lg.rank;
  if (nr <= 0) return cudaSuccess;
  const int64_t total = nr * (a.lg.KC * kKChunk + a.lg.NT * kBN);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  lora_swap_kernel<<<unsigned(blocks), 256, 0, s>>>(a.layer, a.lg, a.A, a.B, a.r_e, a.scale);
  return cudaGetLastError();
}

cudaError_t run_bounded_wait_test(uint64_t timeout_ns, uint32_t* status_out, cudaStream_t s) {
  const uint32_t init = 0xFFFFFFFFu;
  cudaError_t e = cudaMemcpyToSymbolAsync(g_bounded_wait_status, &init, 4, 0, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  bounded_wait_test_kernel<<<1, 32, 0, s>>>(timeout_ns);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaMemcpyFromSymbolAsync(status_out, g_bounded_wait_status, 4, 0, cudaMemcpyDeviceToHost, s)) !=
      cudaSuccess)
    return e;
  return cudaStreamSynchronize(s);
}

}  // namespace svdq
