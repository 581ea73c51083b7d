// blob.cpp -- a prepared layer as one flat, versioned host blob, and back.
//
// The blob is what a checkpoint stores in place of W: the device image in its base state (rank r,
// no adapter) plus the host arrays the exports and a later LoRA swap read.  Importing it gives a
// handle equal to the one that wrote it, with no SVD and no quantization run again.
//
// Layout (little-endian, every section 8-byte aligned):
//   BlobHeader (128 bytes) | image | lambda f32 [K] | 1/lambda f32 [K] | L1 bf16 [K, r] |
//   L2 bf16 [r, N] | sigma f64 [n_sigma]
// The header's checksum is FNV-1a (64-bit) over every byte after the header.
#include <cstring>
#include <new>
#include <string>

#include "layer.h"

namespace {

constexpr char kMagic[8] = {'S', 'V', 'D', 'Q', 'L', 'A', 'Y', 'R'};
constexpr uint32_t kBlobVersion = 1;

struct BlobHeader {
  char magic[8];
  uint32_t version, header_bytes;
  int64_t K, N;
  int32_t rank, rank_capacity, format, has_bias;
  float g_a, g_w, alpha, inv_alpha, c_a;
  uint32_t reserved0;
  uint64_t image_bytes, n_sigma;
  double resid_f64, resid_bf16;
  uint64_t checksum;
  uint8_t reserved1[16];
};
static_assert(sizeof(BlobHeader) == 128, "blob header is 128 bytes");

size_t pad8(size_t n) { return (n + 7) & ~size_t(7); }

uint64_t fnv1a(const uint8_t* p, size_t n) {
  uint64_t h = 0xcbf29ce484222325ull;
  for (size_t i = 0; i < n; ++i) h = (h ^ p[i]) * 0x100000001b3ull;
  return h;
}

struct Sections {
  size_t image, lam, inv_lam, l1, l2, sigma, total;
};

Sections sections(const svdq::LayerGeom& g, uint64_t n_sigma) {
  Sections s{};
  size_t o = sizeof(BlobHeader);
  s.image = o;   o += pad8(g.total);
  s.lam = o;     o += pad8(size_t(g.K) * 4);
  s.inv_lam = o; o += pad8(size_t(g.K) * 4);
  s.l1 = o;      o += pad8(size_t(g.K) * g.rank * 2);
  s.l2 = o;      o += pad8(size_t(g.rank) * g.N * 2);
  s.sigma = o;   o += pad8(size_t(n_sigma) * 8);
  s.total = o;
  return s;
}

}  // namespace

namespace svdq {

size_t blob_bytes(const svdq_layer* L) { return sections(L->g, L->sigma.size()).total; }

svdq_status blob_write(const svdq_layer* L, uint8_t* dst, size_t bytes, std::string* err) {
  const Sections s = sections(L->g, L->sigma.size());
  if (bytes < s.total) return *err = "blob needs " + std::to_string(s.total) + " bytes", SVDQ_ERR_BUFFER_TOO_SMALL;
  std::memset(dst, 0, s.total);
  const LayerGeom& g = L->g;
  std::memcpy(dst + s.image, L->image.data(), g.total);
  std::memcpy(dst + s.lam, L->lam.data(), size_t(g.K) * 4);
  std::memcpy(dst + s.inv_lam, L->inv_lam.data(), size_t(g.K) * 4);
  std::memcpy(dst + s.l1, L->l1.data(), size_t(g.K) * g.rank * 2);
  std::memcpy(dst + s.l2, L->l2.data(), size_t(g.rank) * g.N * 2);
  if (!L->sigma.empty()) std::memcpy(dst + s.sigma, L->sigma.data(), L->sigma.size() * 8);
  BlobHeader h{};
  std::memcpy(h.magic, kMagic, 8);
  h.version = kBlobVersion;
  h.header_bytes = sizeof(BlobHeader);
  h.K = g.K;
  h.N = g.N;
  h.rank = g.rank;
  h.rank_capacity = g.rcap;
  h.format = L->format;
  h.has_bias = L->has_bias ? 1 : 0;
  h.g_a = L->g_a;
  h.g_w = L->g_w;
  h.alpha = L->alpha;
  h.inv_alpha = L->inv_alpha;
  h.c_a = L->c_a;
  h.image_bytes = g.total;
  h.n_sigma = L->sigma.size();
  h.resid_f64 = L->resid_f64;
  h.resid_bf16 = L->resid_bf16;
  h.checksum = fnv1a(dst + sizeof(BlobHeader), s.total - sizeof(BlobHeader));
  std::memcpy(dst, &h, sizeof h);
  return SVDQ_OK;
}

svdq_status blob_read(const uint8_t* src, size_t bytes, svdq_layer** out, std::string* err) {
  if (bytes < sizeof(BlobHeader)) return *err = "blob shorter than its header", SVDQ_ERR_INVALID_ARGUMENT;
  BlobHeader h;
  std::memcpy(&h, src, sizeof h);
  if (std::memcmp(h.magic, kMagic, 8) != 0) return *err = "not a layer blob (magic)", SVDQ_ERR_INVALID_ARGUMENT;
  if (h.version != kBlobVersion || h.header_bytes != sizeof(BlobHeader))
    return *err = "unsupported blob version " + std::to_string(h.version), SVDQ_ERR_INVALID_ARGUMENT;
  if (h.format != SVDQ_FMT_NVFP4 && h.format != SVDQ_FMT_INT4)
    return *err = "unknown format in blob", SVDQ_ERR_INVALID_ARGUMENT;
  if (h.K < 64 || h.N < 64 || h.K % 64 || h.N % 64 || h.K > (int64_t(1) << 24) || h.N > (int64_t(1) << 24) ||
      h.rank < 0 || h.rank % 16 || h.rank_capacity < h.rank || h.rank_capacity % 16 ||
      h.rank_capacity > kMaxRankCapacity || h.rank > h.K || h.rank > h.N)
    return *err = "blob holds an unsupported shape", SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (h.n_sigma != 0 && h.n_sigma != uint64_t(h.rank))
    return *err = "blob holds a wrong number of singular values", SVDQ_ERR_INVALID_ARGUMENT;
  const LayerGeom g = make_layer_geom(h.K, h.N, h.rank, h.rank_capacity);
  if (h.image_bytes != g.total) return *err = "blob image size does not match its shape", SVDQ_ERR_INVALID_ARGUMENT;
  const Sections s = sections(g, h.n_sigma);
  if (bytes < s.total) return *err = "blob is truncated (" + std::to_string(s.total) + " bytes expected)",
                              SVDQ_ERR_INVALID_ARGUMENT;
  if (fnv1a(src + sizeof(BlobHeader), s.total - sizeof(BlobHeader)) != h.checksum)
    return *err = "blob checksum mismatch", SVDQ_ERR_INVALID_ARGUMENT;
  svdq_layer* L = new (std::nothrow) svdq_layer();
  if (!L) return *err = "host allocation failed", SVDQ_ERR_HOST_ALLOC;
  try {
    L->g = g;
    L->format = h.format;
    L->has_bias = h.has_bias != 0;
    L->g_a = h.g_a;
    L->g_w = h.g_w;
    L->alpha = h.alpha;
    L->inv_alpha = h.inv_alpha;
    L->c_a = h.c_a;
    L->resid_f64 = h.resid_f64;
    L->resid_bf16 = h.resid_bf16;
    L->r_tot = g.rank;
    L->image.assign(src + s.image, src + s.image + g.total);
    L->lam.resize(g.K);
    L->inv_lam.resize(g.K);
    std::memcpy(L->lam.data(), src + s.lam, size_t(g.K) * 4);
    std::memcpy(L->inv_lam.data(), src + s.inv_lam, size_t(g.K) * 4);
    L->l1.resize(size_t(g.K) * g.rank);
    L->l2.resize(size_t(g.rank) * g.N);
    std::memcpy(L->l1.data(), src + s.l1, L->l1.size() * 2);
    std::memcpy(L->l2.data(), src + s.l2, L->l2.size() * 2);
    L->sigma.resize(h.n_sigma);
    if (h.n_sigma) std::memcpy(L->sigma.data(), src + s.sigma, h.n_sigma * 8);
  } catch (const std::bad_alloc&) {
    delete L;
    return *err = "host allocation failed", SVDQ_ERR_HOST_ALLOC;
  }
  *out = L;
  return SVDQ_OK;
}

}  // namespace svdq
