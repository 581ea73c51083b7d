// api.cpp -- the extern "C" entry points declared in include/svdq.h.
//
// Argument checking, device checks and marshalling only: the preparation
// lives in prepare.cpp / svd.cpp, the hot path in act_quant.cu and gemm.cu.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <exception>
#include <new>
#include <string>

#include "kernels.h"
#include "layer.h"
#include "int4.h"
#include "w4a16.h"

namespace {

thread_local std::string g_last_error;
std::atomic<int> g_arch_override{0};

svdq_status fail(svdq_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

svdq_status cuda_fail(cudaError_t e, const char* what) {
  std::string m = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return fail(SVDQ_ERR_CUDA, m);
}

// The kernels use tcgen05 / TMA forms that exist on sm_100 only.  Like the
// Nunchaku-Lite loader (Diffusers page, "kernel variants per GPU generation"),
// refuse other devices with a clear error instead of producing wrong output.
svdq_status check_device(int* dev_out, int* sms_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0, sms = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute(major)");
  if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute(minor)");
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
  int sm = major * 10 + minor;
  const int ov = g_arch_override.load();
  if (ov > 0) sm = ov;
  if (sm != 100)
    return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "device " + std::to_string(dev) + " is sm_" + std::to_string(sm) +
                                                 "; these kernels need sm_100 (B200/GB200)");
  if (dev_out) *dev_out = dev;
  if (sms_out) *sms_out = sms;
  return SVDQ_OK;
}

svdq_status check_uploaded(const svdq_layer* L) {
  if (!L) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer is NULL");
  if (!L->dev_buf) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer has not been uploaded (svdq_layer_upload)");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != L->device)
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "current device " + std::to_string(dev) + " differs from the layer's device " +
                                               std::to_string(L->device));
  return SVDQ_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Note that act_buf now holds activations quantized under the handle's current factors.
void note_act(const svdq_layer* L, const void* act_buf) {
  auto& N = L->notes;
  std::lock_guard<std::mutex> lk(N.mu);
  for (auto& n : N.ring)
    if (n.buf == act_buf) {
      n.gen = L->swap_gen;
      return;
    }
  N.ring[N.next] = {act_buf, L->swap_gen};
  N.next = (N.next + 1) % svdq_layer::ActNotes::kSize;
}

// True when act_buf was last quantized through this handle under other low-rank factors.
bool act_is_stale(const svdq_layer* L, const void* act_buf) {
  auto& N = L->notes;
  std::lock_guard<std::mutex> lk(N.mu);
  for (const auto& n : N.ring)
    if (n.buf == act_buf) return n.gen != L->swap_gen;
  return false;
}

}  // namespace

extern "C" {

int svdq_abi_version(void) { return SVDQ_ABI_VERSION; }

const char* svdq_last_error(void) { return g_last_error.c_str(); }

svdq_status svdq_calibrate_amax(const uint16_t* X, int64_t M, int64_t K, float* amax) {
  if (!X || !amax) return fail(SVDQ_ERR_INVALID_ARGUMENT, "X and amax are required");
  if (M < 0 || K < 1) return fail(SVDQ_ERR_INVALID_ARGUMENT, "bad shape");
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      const uint32_t u = uint32_t(X[m * K + k] & 0x7FFFu) << 16;
      float f;
      std::memcpy(&f, &u, 4);
      amax[k] = std::max(amax[k], f);
    }
  return SVDQ_OK;
}

size_t svdq_layer_device_bytes(const svdq_prepare_desc* d) {
  std::string err;
  if (svdq::validate_desc(d, &err) != SVDQ_OK) {
    g_last_error = err;
    return 0;
  }
  return svdq::make_layer_geom(d->K, d->N, d->rank, d->rank_capacity).total;
}

svdq_status svdq_prepare_host(const svdq_prepare_desc* d, svdq_layer** out) {
  std::string err;
  svdq_status st = svdq::prepare_host(d, out, &err);
  if (st != SVDQ_OK) return fail(st, err);
  return SVDQ_OK;
}

svdq_status svdq_layer_upload(svdq_layer* L, void* dev_buf, size_t dev_buf_bytes, void* stream) {
  if (!L || !dev_buf) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer and dev_buf are required");
  if (!aligned(dev_buf, 256)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "dev_buf must be 256-byte aligned");
  if (dev_buf_bytes < L->g.total)
    return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "dev_buf needs " + std::to_string(L->g.total) + " bytes");
  int dev = 0, sms = 0;
  svdq_status st = check_device(&dev, &sms);
  if (st != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(dev_buf, L->image.data(), L->g.total, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(layer image)");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  L->dev_buf = dev_buf;
  L->dev_bytes = dev_buf_bytes;
  L->device = dev;
  L->num_sms = sms;
  L->r_tot = L->g.rank;
  return SVDQ_OK;
}

svdq_status svdq_prepare_weights(const svdq_prepare_desc* d, void* dev_buf, size_t dev_buf_bytes,
                                 svdq_layer** out, void* stream) {
  if (!out) return fail(SVDQ_ERR_INVALID_ARGUMENT, "out is NULL");
  svdq_layer* L = nullptr;
  svdq_status st = svdq_prepare_host(d, &L);
  if (st != SVDQ_OK) return st;
  st = svdq_layer_upload(L, dev_buf, dev_buf_bytes, stream);
  if (st != SVDQ_OK) {
    delete L;
    return st;
  }
  *out = L;
  return SVDQ_OK;
}

svdq_status svdq_act_buffer_bytes(const svdq_layer* L, int64_t M, size_t* bytes) {
  if (!L || !bytes) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer and bytes are required");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARGUMENT, "M must be >= 1");
  *bytes = svdq::make_act_geom(L->g, M).total;
  return SVDQ_OK;
}

svdq_status svdq_quantize_act(const svdq_layer* L, const void* X, int64_t M, void* act_buf, size_t act_buf_bytes,
                              void* stream) {
  svdq_status st = check_uploaded(L);
  if (st != SVDQ_OK) return st;
  if (!X || !act_buf) return fail(SVDQ_ERR_INVALID_ARGUMENT, "X and act_buf are required");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARGUMENT, "M must be >= 1");
  if (!aligned(X, 16)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "X must be 16-byte aligned");
  if (!aligned(act_buf, 256)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "act_buf must be 256-byte aligned");
  const size_t need = svdq::make_act_geom(L->g, M).total;
  if (act_buf_bytes < need) return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "act_buf needs " + std::to_string(need) + " bytes");
  if ((st = check_device(nullptr, nullptr)) != SVDQ_OK) return st;
  svdq::ActQuantLaunch a{};
  a.X = X;
  a.layer = static_cast<const uint8_t*>(L->dev_buf);
  a.act = static_cast<uint8_t*>(act_buf);
  a.lg = L->g;
  a.M = M;
  a.r_tot = L->r_tot;
  a.g_a = L->g_a;
  a.c_a = L->c_a;
  a.inv_alpha = L->inv_alpha;
  a.num_sms = L->num_sms;
  a.timeout_ns = svdq::kDefaultTimeoutNs;
  a.int4 = L->format == SVDQ_FMT_INT4 ? 1 : 0;
  const char* why = "";
  cudaError_t e = svdq::launch_act_quant(a, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) return cuda_fail(e, why);
  note_act(L, act_buf);
  return SVDQ_OK;
}

namespace {

svdq_status linear_launch(const svdq_layer* L, const void* act_buf, size_t act_buf_bytes, int64_t M, void* Y,
                          int epilogue, const svdq::GemmLaunch* qkv, void* stream) {
  svdq_status st = check_uploaded(L);
  if (st != SVDQ_OK) return st;
  if (!act_buf || !Y) return fail(SVDQ_ERR_INVALID_ARGUMENT, "act_buf and Y are required");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARGUMENT, "M must be >= 1");
  if (epilogue != SVDQ_EPI_NONE && epilogue != SVDQ_EPI_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "unknown epilogue");
  if (!aligned(Y, 32)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "Y must be 32-byte aligned");
  if (!aligned(act_buf, 256)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "act_buf must be 256-byte aligned");
  const size_t need = svdq::make_act_geom(L->g, M).total;
  if (act_buf_bytes < need) return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "act_buf needs " + std::to_string(need) + " bytes");
  if (M * L->g.N > (int64_t(1) << 31) * 2 || M > (int64_t(1) << 31) - 1)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "M too large");
  if (act_is_stale(L, act_buf))
    return fail(SVDQ_ERR_INVALID_ARGUMENT,
                "act_buf was quantized before the layer's last LoRA swap; quantize X again (svdq_quantize_act)");
  if ((st = check_device(nullptr, nullptr)) != SVDQ_OK) return st;
  if (L->format == SVDQ_FMT_INT4) {
    if (qkv) return fail(SVDQ_ERR_INVALID_ARGUMENT, "the fused QKV epilogue is built for NVFP4 layers only");
    svdq::Int4GemmLaunch a{};
    a.act = static_cast<const uint8_t*>(act_buf);
    a.layer = static_cast<const uint8_t*>(L->dev_buf);
    a.Y = Y;
    a.lg = L->g;
    a.M = M;
    a.r_tot = L->r_tot;
    a.has_bias = L->has_bias ? 1 : 0;
    a.epilogue = epilogue;
    a.alpha = L->alpha;
    a.pre_a = 1.0f / L->g_a;  // powers of two: exact
    a.pre_w = 1.0f / L->g_w;
    a.num_sms = L->num_sms;
    a.timeout_ns = svdq::kDefaultTimeoutNs;
    const char* why = "";
    cudaError_t e = svdq::launch_gemm_int4(a, static_cast<cudaStream_t>(stream), &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
    return SVDQ_OK;
  }
  svdq::GemmLaunch a = qkv ? *qkv : svdq::GemmLaunch{};
  a.act = static_cast<const uint8_t*>(act_buf);
  a.layer = static_cast<const uint8_t*>(L->dev_buf);
  a.Y = Y;
  a.lg = L->g;
  a.M = M;
  a.r_tot = L->r_tot;
  a.has_bias = L->has_bias ? 1 : 0;
  a.epilogue = epilogue;
  a.alpha = L->alpha;
  a.num_sms = L->num_sms;
  a.timeout_ns = svdq::kDefaultTimeoutNs;
  const char* why = "";
  cudaError_t e = svdq::launch_gemm(a, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) return cuda_fail(e, why);
  return SVDQ_OK;
}

}  // namespace

svdq_status svdq_w4a4_linear(const svdq_layer* L, const void* act_buf, size_t act_buf_bytes, int64_t M, void* Y,
                             int epilogue, void* stream) {
  return linear_launch(L, act_buf, act_buf_bytes, M, Y, epilogue, nullptr, stream);
}

svdq_status svdq_mlp_workspace_bytes(const svdq_layer* fc1, const svdq_layer* fc2, int64_t M, size_t* bytes) {
  if (!fc1 || !fc2 || !bytes) return fail(SVDQ_ERR_INVALID_ARGUMENT, "fc1, fc2 and bytes are required");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARGUMENT, "M must be >= 1");
  if (fc2->g.K != fc1->g.N) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "fc2's K must equal fc1's N");
  *bytes = fc2->r_tot > 0 ? svdq::mlp_partial_bytes(fc1->g.NT, svdq::make_act_geom(fc1->g, M).MT, fc2->r_tot) : 0;
  return SVDQ_OK;
}

svdq_status svdq_w4a4_linear_mlp(const svdq_layer* fc1, const void* act1, size_t act1_bytes, int64_t M,
                                 const svdq_layer* fc2, void* act2, size_t act2_bytes, void* workspace,
                                 size_t workspace_bytes, int epilogue, void* stream) {
  svdq_status st = check_uploaded(fc1);
  if (st != SVDQ_OK) return st;
  if ((st = check_uploaded(fc2)) != SVDQ_OK) return st;
  if (fc1->format != SVDQ_FMT_NVFP4 || fc2->format != SVDQ_FMT_NVFP4)
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "the fused MLP pair is built for NVFP4 layers only");
  if (!act1 || !act2) return fail(SVDQ_ERR_INVALID_ARGUMENT, "act1 and act2 are required");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARGUMENT, "M must be >= 1");
  if (M > (int64_t(1) << 31) - 1) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "M too large");
  if (epilogue != SVDQ_EPI_NONE && epilogue != SVDQ_EPI_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "unknown epilogue");
  if (fc2->g.K != fc1->g.N) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "fc2's K must equal fc1's N");
  if (!aligned(act1, 256) || !aligned(act2, 256))
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "act1 and act2 must be 256-byte aligned");
  const size_t need1 = svdq::make_act_geom(fc1->g, M).total, need2 = svdq::make_act_geom(fc2->g, M).total;
  if (act1_bytes < need1) return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "act1 needs " + std::to_string(need1) + " bytes");
  if (act2_bytes < need2) return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "act2 needs " + std::to_string(need2) + " bytes");
  const svdq::ActGeom ag1 = svdq::make_act_geom(fc1->g, M);
  const size_t needw = fc2->r_tot > 0 ? svdq::mlp_partial_bytes(fc1->g.NT, ag1.MT, fc2->r_tot) : 0;
  if (needw > 0 && !workspace) return fail(SVDQ_ERR_INVALID_ARGUMENT, "workspace is required when fc2 has ranks");
  if (needw > 0 && !aligned(workspace, 16)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "workspace must be 16-byte aligned");
  if (workspace_bytes < needw)
    return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "workspace needs " + std::to_string(needw) + " bytes");
  if (act_is_stale(fc1, act1))
    return fail(SVDQ_ERR_INVALID_ARGUMENT,
                "act1 was quantized before fc1's last LoRA swap; quantize X again (svdq_quantize_act)");
  if ((st = check_device(nullptr, nullptr)) != SVDQ_OK) return st;
  svdq::GemmLaunch a{};
  a.act = static_cast<const uint8_t*>(act1);
  a.layer = static_cast<const uint8_t*>(fc1->dev_buf);
  a.Y = nullptr;
  a.lg = fc1->g;
  a.M = M;
  a.r_tot = fc1->r_tot;
  a.has_bias = fc1->has_bias ? 1 : 0;
  a.epilogue = epilogue;
  a.alpha = fc1->alpha;
  a.num_sms = fc1->num_sms;
  a.timeout_ns = svdq::kDefaultTimeoutNs;
  a.mlp_act2 = static_cast<uint8_t*>(act2);
  a.mlp_layer2 = static_cast<const uint8_t*>(fc2->dev_buf);
  a.mlp_lg2 = fc2->g;
  a.mlp_r2 = fc2->r_tot;
  a.mlp_g_a2 = fc2->g_a;
  a.mlp_c_a2 = fc2->c_a;
  a.mlp_partial = static_cast<float*>(workspace);
  const char* why = "";
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = svdq::launch_gemm(a, s, &why);
  if (e != cudaSuccess) return cuda_fail(e, why);
  if (fc2->r_tot > 0) {
    const svdq::ActGeom ag2 = svdq::make_act_geom(fc2->g, M);
    svdq::MlpReduceLaunch r{};
    r.partial = static_cast<const float*>(workspace);
    r.nt = int32_t(fc1->g.NT);
    r.rows = ag1.MT * svdq::kBM;
    r.r2 = fc2->r_tot;
    r.inv_alpha2 = fc2->inv_alpha;
    r.lr2 = static_cast<uint8_t*>(act2) + ag2.off_lr;
    r.RJ2 = int32_t(ag2.RJ);
    e = svdq::launch_mlp_reduce(r, s);
    if (e != cudaSuccess) return cuda_fail(e, "launch of the MLP partial reduction failed");
  }
  note_act(fc2, act2);
  return SVDQ_OK;
}

svdq_status svdq_w4a4_linear_mlp_static(const svdq_layer* fc1, const void* act1, size_t act1_bytes, int64_t M,
                                        const svdq_layer* fc2, void* act2, size_t act2_bytes, int epilogue,
                                        void* stream) {
  if (!fc1 || !fc2) return fail(SVDQ_ERR_INVALID_ARGUMENT, "fc1 and fc2 are required");
  size_t need = 0;
  svdq_status st = svdq_mlp_workspace_bytes(fc1, fc2, M, &need);
  if (st != SVDQ_OK) return st;
  if (need > svdq::kMlpStaticBytes)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE,
                "this pair needs " + std::to_string(need) + " bytes of scratch; the library's static area holds " +
                    std::to_string(svdq::kMlpStaticBytes) + " (pass a workspace to svdq_w4a4_linear_mlp)");
  if ((st = check_uploaded(fc1)) != SVDQ_OK) return st;
  void* scratch = nullptr;
  cudaError_t e = svdq::mlp_static_scratch(fc1->device, &scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(the static MLP scratch)");
  return svdq_w4a4_linear_mlp(fc1, act1, act1_bytes, M, fc2, act2, act2_bytes, scratch, svdq::kMlpStaticBytes,
                              epilogue, stream);
}

svdq_status svdq_rope_packed_bytes(int64_t M, int32_t head_dim, size_t* bytes) {
  if (!bytes) return fail(SVDQ_ERR_INVALID_ARGUMENT, "bytes is required");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARGUMENT, "M must be >= 1");
  if (head_dim != svdq::kRopeHeadDim) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "head_dim must be 128");
  *bytes = svdq::rope_packed_bytes(M);
  return SVDQ_OK;
}

svdq_status svdq_rope_pack(const void* rope, int64_t M, int32_t head_dim, void* packed, size_t packed_bytes,
                           void* stream) {
  size_t need = 0;
  svdq_status st = svdq_rope_packed_bytes(M, head_dim, &need);
  if (st != SVDQ_OK) return st;
  if (!rope || !packed) return fail(SVDQ_ERR_INVALID_ARGUMENT, "rope and packed are required");
  if (!aligned(rope, 16) || !aligned(packed, 16))
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "rope and packed must be 16-byte aligned");
  if (packed_bytes < need)
    return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "packed needs " + std::to_string(need) + " bytes");
  if ((st = check_device(nullptr, nullptr)) != SVDQ_OK) return st;
  cudaError_t e = svdq::launch_rope_pack(static_cast<const float*>(rope), M, static_cast<float*>(packed),
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "launch of the rotary table pack kernel");
  return SVDQ_OK;
}

svdq_status svdq_w4a4_linear_qkv_norm_rope(const svdq_layer* L, const void* act_buf, size_t act_buf_bytes,
                                           int64_t M, void* Y, const void* norm_q, const void* norm_k,
                                           const void* rope_packed, size_t rope_packed_bytes, int32_t head_dim,
                                           float eps, void* stream) {
  svdq_status st = check_uploaded(L);
  if (st != SVDQ_OK) return st;
  if (L->format != SVDQ_FMT_NVFP4)
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "the fused QKV epilogue is built for NVFP4 layers only");
  if (head_dim != svdq::kRopeHeadDim) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "head_dim must be 128");
  if (L->g.N % 3 || (L->g.N / 3) % head_dim)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "N must be 3 x a multiple of head_dim (Q | K | V)");
  if (!norm_q || !norm_k || !rope_packed)
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "norm_q, norm_k and rope_packed are required");
  if (!aligned(norm_q, 16) || !aligned(norm_k, 16) || !aligned(rope_packed, 16))
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "norm_q, norm_k and rope_packed must be 16-byte aligned");
  if (M >= 1 && rope_packed_bytes < svdq::rope_packed_bytes(M))
    return fail(SVDQ_ERR_BUFFER_TOO_SMALL,
                "rope_packed needs " + std::to_string(svdq::rope_packed_bytes(M)) + " bytes (svdq_rope_pack)");
  if (!std::isfinite(eps) || eps < 0.0f) return fail(SVDQ_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
  svdq::GemmLaunch q{};
  q.qkv_cols = int32_t(L->g.N / 3);
  q.norm_q = static_cast<const uint16_t*>(norm_q);
  q.norm_k = static_cast<const uint16_t*>(norm_k);
  q.rope = static_cast<const float*>(rope_packed);
  q.eps = eps;
  return linear_launch(L, act_buf, act_buf_bytes, M, Y, SVDQ_EPI_NONE, &q, stream);
}

svdq_status svdq_lora_swap(svdq_layer* L, const void* A, const void* B, int32_t r_e, float scale, void* stream) {
  if (!L) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer is NULL");
  if (r_e < 0 || r_e % 16) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "LoRA rank must be a multiple of 16");
  if (r_e > L->g.rcap - L->g.rank)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "rank + LoRA rank exceeds rank_capacity (" + std::to_string(L->g.rcap) + ")");
  if (r_e > 0 && (!A || !B)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "A and B are required");
  if (r_e > 0 && (!aligned(A, 2) || !aligned(B, 2)))
    return fail(SVDQ_ERR_INVALID_ARGUMENT, "A and B must be 2-byte aligned (bf16 elements)");
  if (!std::isfinite(scale)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "scale must be finite");
  svdq_status st = check_uploaded(L);
  if (st != SVDQ_OK) return st;
  svdq::LoraLaunch a{};
  a.layer = static_cast<uint8_t*>(L->dev_buf);
  a.lg = L->g;
  a.A = static_cast<const uint16_t*>(A);
  a.B = static_cast<const uint16_t*>(B);
  a.r_e = r_e;
  a.scale = scale;
  cudaError_t e = svdq::launch_lora_swap(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "launch of the LoRA swap kernel");
  L->r_tot = L->g.rank + r_e;
  ++L->swap_gen;
  return SVDQ_OK;
}

svdq_status svdq_layer_export(const svdq_layer* L, int what, void* host_dst, size_t bytes) {
  if (!L || !host_dst) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer and host_dst are required");
  std::string err;
  svdq_status st = svdq::export_array(L, what, host_dst, bytes, &err);
  if (st != SVDQ_OK) return fail(st, err);
  return SVDQ_OK;
}

svdq_status svdq_act_unpack(const svdq_layer* L, int64_t M, const void* act_host, size_t bytes, uint8_t* codes,
                            uint8_t* scales, uint16_t* lr) {
  if (!L || !act_host) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer and act_host are required");
  if (M < 1) return fail(SVDQ_ERR_INVALID_ARGUMENT, "M must be >= 1");
  std::string err;
  svdq_status st = svdq::act_unpack(L, M, static_cast<const uint8_t*>(act_host), bytes, codes, scales, lr, &err);
  if (st != SVDQ_OK) return fail(st, err);
  return SVDQ_OK;
}

svdq_status svdq_get_layer_info(const svdq_layer* L, svdq_layer_info* info) {
  if (!L || !info) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer and info are required");
  info->K = L->g.K;
  info->N = L->g.N;
  info->rank = L->g.rank;
  info->rank_total = L->r_tot;
  info->rank_capacity = L->g.rcap;
  info->format = L->format;
  info->g_a = L->g_a;
  info->g_w = L->g_w;
  info->alpha = L->alpha;
  info->device_bytes = L->g.total;
  info->dev_buf = L->dev_buf;
  info->device = L->device;
  return SVDQ_OK;
}

svdq_status svdq_poll_status(const svdq_layer* L, void* stream) {
  svdq_status st = check_uploaded(L);
  if (st != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  uint8_t* status = static_cast<uint8_t*>(L->dev_buf) + L->g.off_status;
  cudaError_t e = cudaMemcpyAsync(&word, status, 4, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(status)");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  if (word == 0) return SVDQ_OK;
  if ((e = cudaMemsetAsync(status, 0, 4, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  char buf[96];
  std::snprintf(buf, sizeof buf, "a kernel gave up a bounded wait (status word 0x%x)", word);
  return fail(SVDQ_ERR_TIMEOUT, buf);
}

void svdq_layer_destroy(svdq_layer* L) { delete L; }

svdq_status svdq_layer_clone(const svdq_layer* L, svdq_layer** out) {
  if (!L || !out) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer and out are required");
  svdq_layer* c = nullptr;
  try {
    c = new svdq_layer(*L);
  } catch (const std::bad_alloc&) {
    return fail(SVDQ_ERR_HOST_ALLOC, "host allocation failed while copying the layer");
  }
  c->dev_buf = nullptr;
  c->dev_bytes = 0;
  c->device = -1;
  c->num_sms = 0;
  c->r_tot = c->g.rank;
  *out = c;
  return SVDQ_OK;
}

svdq_status svdq_layer_serialize(const svdq_layer* L, void* host_dst, size_t bytes, size_t* bytes_needed) {
  if (!L) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer is NULL");
  const size_t need = svdq::blob_bytes(L);
  if (bytes_needed) *bytes_needed = need;
  if (!host_dst) {
    if (!bytes_needed) return fail(SVDQ_ERR_INVALID_ARGUMENT, "give host_dst or bytes_needed");
    return SVDQ_OK;
  }
  std::string err;
  svdq_status st = svdq::blob_write(L, static_cast<uint8_t*>(host_dst), bytes, &err);
  if (st != SVDQ_OK) return fail(st, err);
  return SVDQ_OK;
}

svdq_status svdq_layer_import(const void* blob, size_t bytes, svdq_layer** out) {
  if (!blob || !out) return fail(SVDQ_ERR_INVALID_ARGUMENT, "blob and out are required");
  std::string err;
  svdq_status st = svdq::blob_read(static_cast<const uint8_t*>(blob), bytes, out, &err);
  if (st != SVDQ_OK) return fail(st, err);
  return SVDQ_OK;
}

void svdq_test_override_device_arch(int sm) { g_arch_override.store(sm); }

svdq_status svdq_test_bounded_wait(uint64_t timeout_ns, uint32_t* status_out, void* stream) {
  if (!status_out) return fail(SVDQ_ERR_INVALID_ARGUMENT, "status_out is NULL");
  svdq_status st = check_device(nullptr, nullptr);
  if (st != SVDQ_OK) return st;
  cudaError_t e = svdq::run_bounded_wait_test(timeout_ns, status_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bounded-wait test kernel");
  return SVDQ_OK;
}


// ------------------------------------------------------------------ W4A16
size_t svdq_w4a16_device_bytes(const svdq_w4a16_desc* d) {
  if (!d || d->K < 64 || d->K % 64 || d->K > 12288 || d->N < 1 || d->N > (int64_t(1) << 24)) {
    g_last_error = "bad W4A16 descriptor";
    return 0;
  }
  return svdq::make_w4a16_geom(d->K, d->N).total;
}

svdq_status svdq_w4a16_prepare_host(const svdq_w4a16_desc* d, svdq_w4a16** out) {
  if (!out) return fail(SVDQ_ERR_INVALID_ARGUMENT, "out is NULL");
  std::string err;
  auto* L = new (std::nothrow) svdq_w4a16();
  if (!L) return fail(SVDQ_ERR_HOST_ALLOC, "host allocation failed");
  svdq_status st;
  try {
    st = svdq::w4a16_quantize(d, &L->image, &L->codes, &L->scales, &L->gscale, &err);
  } catch (const std::bad_alloc&) {
    st = SVDQ_ERR_HOST_ALLOC;
    err = "host allocation failed while quantizing the W4A16 layer";
  } catch (const std::exception& e) {
    st = SVDQ_ERR_INTERNAL;
    err = std::string("W4A16 quantization failed: ") + e.what();
  }
  if (st != SVDQ_OK) {
    delete L;
    return fail(st, err);
  }
  L->g = svdq::make_w4a16_geom(d->K, d->N);
  L->has_bias = d->bias != nullptr;
  *out = L;
  return SVDQ_OK;
}

svdq_status svdq_w4a16_upload(svdq_w4a16* L, void* dev_buf, size_t dev_buf_bytes, void* stream) {
  if (!L || !dev_buf) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer and dev_buf are required");
  if (!aligned(dev_buf, 256)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "dev_buf must be 256-byte aligned");
  if (dev_buf_bytes < L->g.total)
    return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "dev_buf needs " + std::to_string(L->g.total) + " bytes");
  int dev = 0, sms = 0;
  svdq_status st = check_device(&dev, &sms);
  if (st != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(dev_buf, L->image.data(), L->g.total, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(W4A16 image)");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  L->dev_buf = dev_buf;
  L->device = dev;
  L->num_sms = sms;
  return SVDQ_OK;
}

svdq_status svdq_w4a16_linear(const svdq_w4a16* L, const void* X, int64_t M, void* Y, void* stream) {
  if (!L) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer is NULL");
  if (!L->dev_buf) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer is not uploaded to a device");
  if (!X || !Y) return fail(SVDQ_ERR_INVALID_ARGUMENT, "X and Y are required");
  if (M < 1 || M > (int64_t(1) << 31) / L->g.N) return fail(SVDQ_ERR_INVALID_ARGUMENT, "M out of range");
  if (!aligned(X, 16)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "X must be 16-byte aligned");
  if (!aligned(Y, 2)) return fail(SVDQ_ERR_INVALID_ARGUMENT, "Y must be 2-byte aligned");
  svdq_status st = check_device(nullptr, nullptr);
  if (st != SVDQ_OK) return st;
  svdq::W4A16Launch a{};
  a.layer = static_cast<const uint8_t*>(L->dev_buf);
  a.g = L->g;
  a.X = static_cast<const uint16_t*>(X);
  a.M = M;
  a.Y = static_cast<uint16_t*>(Y);
  a.gscale = L->gscale;
  a.has_bias = L->has_bias ? 1 : 0;
  a.num_sms = L->num_sms;
  a.timeout_ns = svdq::kDefaultTimeoutNs;
  const char* why = "";
  cudaError_t e = svdq::launch_w4a16(a, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) return cuda_fail(e, why);
  return SVDQ_OK;
}

svdq_status svdq_w4a16_export(const svdq_w4a16* L, int what, void* host_dst, size_t bytes) {
  if (!L || !host_dst) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer and host_dst are required");
  const auto& g = L->g;
  const uint8_t* img = L->image.data();
  const void* src = nullptr;
  size_t n = 0;
  switch (what) {
    case SVDQ_EXPORT_W_CODES: src = L->codes.data(); n = L->codes.size(); break;
    case SVDQ_EXPORT_W_SCALES: src = L->scales.data(); n = L->scales.size(); break;
    case SVDQ_EXPORT_INV_LAMBDA: src = img + g.off_inv_s; n = size_t(g.K) * 4; break;
    case SVDQ_EXPORT_SCALARS: src = &L->gscale; n = 4; break;
    default: return fail(SVDQ_ERR_INVALID_ARGUMENT, "unknown export for a W4A16 layer");
  }
  if (bytes < n) return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "export needs " + std::to_string(n) + " bytes");
  std::memcpy(host_dst, src, n);
  return SVDQ_OK;
}

svdq_status svdq_w4a16_poll_status(const svdq_w4a16* L, void* stream) {
  if (!L) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer is NULL");
  if (!L->dev_buf) return fail(SVDQ_ERR_INVALID_ARGUMENT, "layer is not uploaded to a device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  uint8_t* status = static_cast<uint8_t*>(L->dev_buf);  // the image's first word
  cudaError_t e = cudaMemcpyAsync(&word, status, 4, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(status)");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  if (word == 0) return SVDQ_OK;
  if ((e = cudaMemsetAsync(status, 0, 4, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  char buf[96];
  std::snprintf(buf, sizeof buf, "the W4A16 kernel gave up a bounded wait (status word 0x%x)", word);
  return fail(SVDQ_ERR_TIMEOUT, buf);
}

void svdq_w4a16_destroy(svdq_w4a16* L) { delete L; }

}  // extern "C"
