// mlp_static.cu -- the fused MLP pair for callers that cannot allocate device memory.
//
// svdq_w4a4_linear_mlp needs a scratch buffer for its float partials of x_hat2 L1_2.  Some
// callers cannot provide one: code that runs where cudaMalloc is not allowed (inside a stream
// capture that must not allocate, under an allocator that owns all device memory, in a plugin
// that is handed only input and output pointers).  For them the library keeps one scratch area
// of kMlpStaticBytes in a file-scope __device__ array: every GPU that loads the library holds it
// until the process exits.  Its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current (a host-side use of the array's name is not a
// device address).
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "kernels.h"

namespace svdq {

namespace {

__device__ __align__(256) unsigned char g_mlp_scratch[kMlpStaticBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64];

}  // namespace

cudaError_t mlp_static_scratch(int dev, void** ptr) {
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_mlp_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace svdq
