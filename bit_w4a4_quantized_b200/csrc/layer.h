// layer.h -- the host-side handle of one prepared layer (internal to the library).
#pragma once

#include <stdint.h>

#include <mutex>
#include <string>
#include <vector>

#include "../../include/svdq.h"
#include "layout.h"

struct svdq_layer {
  svdq::LayerGeom g{};
  int32_t format = SVDQ_FMT_NVFP4;
  std::vector<uint8_t> image;  // device image in its base state (rank r, no adapter)
  std::vector<float> lam, inv_lam;
  std::vector<uint16_t> l1, l2;  // base factors, bf16 [K, r] and [r, N]
  std::vector<float> r32;        // R as float [K, N] (kept only when asked)
  std::vector<double> sigma;     // singular values (library SVD only)
  double resid_f64 = -1.0, resid_bf16 = -1.0;
  float g_a = 1.f, g_w = 1.f, alpha = 1.f, inv_alpha = 1.f, c_a = 1.f;
  int32_t r_tot = 0;  // ranks in use: base rank + attached adapter rank
  // Which low-rank factors the activation buffers were last filled under.  Every LoRA swap
  // bumps swap_gen; svdq_quantize_act notes (buffer, swap_gen) in a small ring, and the
  // linear calls refuse a noted buffer whose generation differs from the handle's, since its
  // lr' columns were computed with the factors the swap replaced.  A copy of the handle
  // starts with no notes.
  struct ActNotes {
    static constexpr int kSize = 64;
    struct Note {
      const void* buf = nullptr;
      uint64_t gen = 0;
    };
    std::mutex mu;
    Note ring[kSize];
    int next = 0;
    ActNotes() = default;
    ActNotes(const ActNotes&) {}
    ActNotes& operator=(const ActNotes&) { return *this; }
  };
  mutable ActNotes notes;
  uint64_t swap_gen = 0;
  bool has_bias = false;
  // device state (after upload)
  void* dev_buf = nullptr;
  size_t dev_bytes = 0;
  int device = -1;
  int num_sms = 0;
};

namespace svdq {

// Host preparation (prepare.cpp).  Returns SVDQ_OK or an error with message.
svdq_status prepare_host(const svdq_prepare_desc* d, svdq_layer** out, std::string* err);
svdq_status validate_desc(const svdq_prepare_desc* d, std::string* err);

// Logical views of the image / of an activation buffer (prepare.cpp).
svdq_status export_array(const svdq_layer* L, int what, void* dst, size_t bytes, std::string* err);
// The flat, versioned blob of a prepared layer (blob.cpp).
size_t blob_bytes(const svdq_layer* L);
svdq_status blob_write(const svdq_layer* L, uint8_t* dst, size_t bytes, std::string* err);
svdq_status blob_read(const uint8_t* src, size_t bytes, svdq_layer** out, std::string* err);

svdq_status act_unpack(const svdq_layer* L, int64_t M, const uint8_t* act, size_t bytes, uint8_t* codes,
                       uint8_t* scales, uint16_t* lr, std::string* err);

}  // namespace svdq
