// prepare.cpp -- offline preparation of one SVDQuant layer on the host.
//
// SVDQuant summary page (hoonably.github.io/blog/svdquant):
//   section 4.2 "Migrate outliers from activation to weight": per-channel
//     smoothing X_hat = X diag(lambda)^-1, W_hat^T = diag(lambda) W^T, with
//     lambda_j = sqrt(max|X_j| / max|W_:,j|) (migration strength 1/2);
//   section 4.2 "Absorb magnified weight outliers with a low-rank branch":
//     W_hat = L1 L2 + R, L1 = U_r Sigma_r, L2 = V_r^T, R quantized to 4 bits;
//   section 3 "Quantization preliminary": Q_X = round(X / s_X),
//     s_X = max|X| / q_max, q_max = 6 for FP4 -- applied per 16-element block
//     with an E4M3 block scale under a float32 tensor scale (NVFP4).
// Every decision that fixes a code is taken in float32 with correctly rounded
// operations, so the codes equal those of any other exact implementation.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <exception>
#include <memory>
#include <new>
#include <thread>

#include "int4.h"
#include "layer.h"
#include "parallel.h"
#include "svd.h"
#include "w4a16.h"

namespace svdq {

namespace {

// ------------------------------------------------------------- number formats
inline float bf16_bits_to_f32(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
// float -> bf16 bits, round to nearest even (finite inputs)
inline uint16_t f32_to_bf16_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}
// double -> bf16 bits directly (8 significant bits, ties to even); subnormal
// results (|x| < 2^-126) round on the 2^-133 grid.
uint16_t f64_to_bf16_bits(double x) {
  if (std::fabs(x) < 0x1p-126) {
    double q = std::nearbyint(x / 0x1p-133);  // current mode: nearest even
    float f = float(q * 0x1p-133);            // exact: a bf16 subnormal fits float
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return uint16_t(u >> 16);
  }
  uint64_t u;
  std::memcpy(&u, &x, 8);
  u += ((uint64_t(1) << 44) - 1) + ((u >> 45) & 1);
  u &= ~((uint64_t(1) << 45) - 1);
  double r;
  std::memcpy(&r, &u, 8);
  float f = float(r);  // exact: 8 significant bits within float range
  uint32_t w;
  std::memcpy(&w, &f, 4);
  return uint16_t(w >> 16);
}

// E4M3 code of a non-negative float: round to nearest even on the E4M3 grid,
// saturating at 448.  The quantum of binade [2^E, 2^(E+1)) is 2^(E-3); the
// subnormal range shares the quantum 2^-9 of the first normal binade.
uint8_t e4m3_code(float v) {
  if (!(v > 0.0f)) return 0;
  if (v >= 448.0f) return 0x7E;
  int e;
  std::frexp(v, &e);  // v in [2^(e-1), 2^e)
  int E = std::max(e - 1, -6);
  float scaled = std::ldexp(v, 3 - E);       // exact power-of-two scaling
  int m = int(std::nearbyint(scaled));       // ties to even
  if (m == 0) return 0;
  if (m >= 16) {
    m = 8;
    E += 1;
  }
  if (E == -6 && m < 8) return uint8_t(m);  // subnormal: exponent field 0
  int code = ((E + 7) << 3) | (m - 8);
  return uint8_t(std::min(code, 0x7E));
}
inline float e4m3_value(uint8_t c) {
  int e = (c >> 3) & 15, m = c & 7;
  return e ? std::ldexp(1.0f + m / 8.0f, e - 7) : std::ldexp(float(m), -9);
}
// E2M1 code (sign in bit 3) of a float: nearest even on {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating.
// The magnitude code counts the decision boundaries passed: the midpoints of the
// grid, each tie going to the even code (0.25 -> 0, 0.75 -> 2, 1.25 -> 2,
// 1.75 -> 4, 2.5 -> 4, 3.5 -> 6, 5 -> 6), and everything above 5 to 7.
inline uint8_t e2m1_code(float t) {
  const uint8_t sign = std::signbit(t) ? 0x8 : 0x0;
  const float a = std::fabs(t);
  const int m = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return sign | uint8_t(m);
}

float global_scale(float amax) { return amax == 0.0f ? 1.0f : amax / 2688.0f; }

// Quantize one row of `k` floats; codes are written through `put_code(k, code)`
// (k even covers a byte pair) and scales through `put_scale(s, code)`.
template <class PutByte, class PutScale>
void quantize_row(const float* t, int64_t k, float g, float c, PutByte&& put_byte, PutScale&& put_scale) {
  for (int64_t b = 0; b < k; b += 16) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(t[b + i]));
    const float prod = amax * c;
    const uint8_t s = e4m3_code(prod);
    const float d = e4m3_value(s) * g;
    const float rcp = (d == 0.0f) ? 0.0f : 1.0f / d;
    for (int i = 0; i < 16; i += 2) {
      const float v0 = t[b + i] * rcp, v1 = t[b + i + 1] * rcp;
      put_byte(b + i, uint8_t(e2m1_code(v0) | (e2m1_code(v1) << 4)));
    }
    put_scale(b / 16, s);
  }
}

// INT4: per group of 64, s = bf16(f32(amax / 7)), rcp = f32(1 / s) (0 when s is
// 0), q = clamp(rne(f32(t * rcp)), -7, 7); codes through `put_byte(k, byte)`
// (two's-complement nibbles, element k even in the low nibble), scales through
// `put_scale(c, bf16 bits)`.  Returns the row's largest scale value.
template <class PutByte, class PutScale>
float quantize_row_int4(const float* t, int64_t k, PutByte&& put_byte, PutScale&& put_scale) {
  float smax = 0.0f;
  for (int64_t b = 0; b < k; b += kGroup4) {
    float amax = 0.0f;
    for (int i = 0; i < kGroup4; ++i) amax = std::max(amax, std::fabs(t[b + i]));
    const uint16_t sb = f32_to_bf16_bits(amax / 7.0f);
    const float s = bf16_bits_to_f32(sb);
    const float rcp = s == 0.0f ? 0.0f : 1.0f / s;
    for (int i = 0; i < kGroup4; i += 2) {
      const float q0 = std::min(7.0f, std::max(-7.0f, std::nearbyint(t[b + i] * rcp)));
      const float q1 = std::min(7.0f, std::max(-7.0f, std::nearbyint(t[b + i + 1] * rcp)));
      put_byte(b + i, uint8_t((int(q0) & 0xF) | ((int(q1) & 0xF) << 4)));
    }
    put_scale(b / kGroup4, sb);
    smax = std::max(smax, s);
  }
  return smax;
}

// The power of two 2^e with v 2^e <= 2^top (and > 2^(top - 1)); 0 for v = 0.
int pow2_exponent(double v, int top) {
  if (!(v > 0.0)) return 0;
  int e;
  std::frexp(v, &e);  // v <= 2^e
  return std::min(100, std::max(-100, top - e));
}

}  // namespace

svdq_status validate_desc(const svdq_prepare_desc* d, std::string* err) {
  if (!d) return *err = "descriptor is NULL", SVDQ_ERR_INVALID_ARGUMENT;
  if (!d->W || !d->act_amax) return *err = "W and act_amax are required", SVDQ_ERR_INVALID_ARGUMENT;
  if (d->format != SVDQ_FMT_NVFP4 && d->format != SVDQ_FMT_INT4)
    return *err = "format must be SVDQ_FMT_NVFP4 or SVDQ_FMT_INT4", SVDQ_ERR_INVALID_ARGUMENT;
  if ((d->L1 == nullptr) != (d->L2 == nullptr))
    return *err = "give both L1 and L2 or neither", SVDQ_ERR_INVALID_ARGUMENT;
  if (d->K < 64 || d->N < 64 || d->K % 64 || d->N % 64)
    return *err = "K and N must be positive multiples of 64", SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (d->K > (int64_t(1) << 24) || d->N > (int64_t(1) << 24))
    return *err = "K and N must be at most 2^24", SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (d->rank < 0 || d->rank % 16) return *err = "rank must be a multiple of 16", SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (d->rank_capacity < d->rank || d->rank_capacity % 16 || d->rank_capacity > kMaxRankCapacity)
    return *err = "rank_capacity must be a multiple of 16 in [rank, 256]", SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (d->rank > std::min(d->K, d->N)) return *err = "rank exceeds min(K, N)", SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (d->svd_power_iters < 0 || d->svd_oversample < 0)
    return *err = "svd parameters must be non-negative", SVDQ_ERR_INVALID_ARGUMENT;
  for (int64_t k = 0; k < d->K; ++k)  // lambda and the activation tensor scale come from these
    if (!(d->act_amax[k] >= 0.0f) || !std::isfinite(d->act_amax[k]))
      return *err = "act_amax[" + std::to_string(k) + "] must be finite and >= 0", SVDQ_ERR_INVALID_ARGUMENT;
  return SVDQ_OK;
}

svdq_status prepare_host(const svdq_prepare_desc* d, svdq_layer** out, std::string* err) {
  svdq_status st = validate_desc(d, err);
  if (st != SVDQ_OK) return st;
  if (!out) return *err = "out is NULL", SVDQ_ERR_INVALID_ARGUMENT;
  const int64_t K = d->K, N = d->N;
  const int r = d->rank;
  int threads = d->num_threads > 0 ? d->num_threads : int(std::max(1u, std::thread::hardware_concurrency()));
  std::unique_ptr<svdq_layer> L(new (std::nothrow) svdq_layer());
  if (!L) return *err = "host allocation failed", SVDQ_ERR_HOST_ALLOC;
  try {
    L->g = make_layer_geom(K, N, r, d->rank_capacity);
    L->format = d->format;
    L->r_tot = r;
    L->has_bias = d->bias != nullptr;
    const LayerGeom& g = L->g;

    // 1. per-input-channel maxima and smoothing factors (float32, correctly rounded)
    std::vector<float> w_amax(K, 0.0f);
    for (int64_t n = 0; n < N; ++n) {
      const uint16_t* w = d->W + n * K;
      for (int64_t k = 0; k < K; ++k) w_amax[k] = std::max(w_amax[k], std::fabs(bf16_bits_to_f32(w[k])));
    }
    L->lam.resize(K);
    L->inv_lam.resize(K);
    for (int64_t k = 0; k < K; ++k) {
      const float a = d->act_amax[k], w = w_amax[k];
      const bool ok = a > 0.0f && w > 0.0f;
      const float lam = ok ? std::sqrt(a / w) : 1.0f;
      L->lam[k] = lam;
      L->inv_lam[k] = 1.0f / lam;
    }

    // 2. smoothed weight W_hat^T [K, N] in float64 (exact: float32 x bf16).
    //    The buffer is left uninitialised (every element is written below, by
    //    the thread that owns its rows).  The transpose goes through 64 x 64
    //    tiles in a local buffer, so that W and R are both walked along rows:
    //    R's row stride is often a multiple of 4 KB, and walking down its
    //    columns would keep evicting lines that map to the same cache sets.
    std::unique_ptr<double[]> r_buf(new double[size_t(K) * N]);
    double* R = r_buf.get();
    parallel_for(ceil_div(K, 64), threads, [&](int64_t b0, int64_t b1) {
      float tile[64][64];
      for (int64_t kb = b0 * 64; kb < std::min(K, b1 * 64); kb += 64) {
        const int64_t kn = std::min<int64_t>(64, K - kb);
        for (int64_t nb = 0; nb < N; nb += 64) {
          const int64_t nn = std::min<int64_t>(64, N - nb);
          for (int64_t j = 0; j < nn; ++j) {
            const uint16_t* w = d->W + (nb + j) * K + kb;
            for (int64_t i = 0; i < kn; ++i) tile[i][j] = bf16_bits_to_f32(w[i]);
          }
          for (int64_t i = 0; i < kn; ++i) {
            const double lam = L->lam[kb + i];
            double* row = R + size_t(kb + i) * N + nb;
            for (int64_t j = 0; j < nn; ++j) row[j] = lam * double(tile[i][j]);
          }
        }
      }
    });

    // 3. low-rank factors, bf16 [K, r] and [r, N]
    L->l1.assign(size_t(K) * r, 0);
    L->l2.assign(size_t(r) * N, 0);
    if (r > 0 && d->L1) {
      std::memcpy(L->l1.data(), d->L1, sizeof(uint16_t) * L->l1.size());
      std::memcpy(L->l2.data(), d->L2, sizeof(uint16_t) * L->l2.size());
    } else if (r > 0) {
      SvdFactors f;
      randomized_svd(R, K, N, r, d->svd_oversample ? d->svd_oversample : 16,
                     d->svd_power_iters ? d->svd_power_iters : 8, d->svd_seed, threads, &f);
      L->sigma = f.sigma;
      std::vector<double> l1d(size_t(K) * r);
      for (int64_t k = 0; k < K; ++k)
        for (int i = 0; i < r; ++i) {
          l1d[size_t(k) * r + i] = f.U[size_t(k) * r + i] * f.sigma[i];
          L->l1[size_t(k) * r + i] = f64_to_bf16_bits(l1d[size_t(k) * r + i]);
        }
      for (size_t i = 0; i < L->l2.size(); ++i) L->l2[i] = f64_to_bf16_bits(f.Vt[i]);
      // ||W_hat^T - L1 L2|| with the float64 factors
      std::vector<double> part(K, 0.0);
      parallel_for(K, threads, [&](int64_t k0, int64_t k1) {
        std::vector<double> row(N);
        for (int64_t k = k0; k < k1; ++k) {
          std::memcpy(row.data(), &R[size_t(k) * N], sizeof(double) * N);
          for (int i = 0; i < r; ++i) {
            const double a = l1d[size_t(k) * r + i];
            const double* v = &f.Vt[size_t(i) * N];
            for (int64_t n = 0; n < N; ++n) row[n] -= a * v[n];
          }
          double s = 0;
          for (int64_t n = 0; n < N; ++n) s += row[n] * row[n];
          part[k] = s;
        }
      });
      double s = 0;
      for (double v : part) s += v;
      L->resid_f64 = std::sqrt(s);
    }

    // 4. residual R = W_hat^T - L1 L2 with the bf16 factors, rank-one terms in
    //    order i = 0 .. r-1 (each product of two bf16 values is exact), and
    //    its squared norm per row, summed over the rows in order afterwards
    std::vector<double> l2d(size_t(r) * N);
    for (size_t i = 0; i < l2d.size(); ++i) l2d[i] = bf16_bits_to_f32(L->l2[i]);
    std::vector<double> row_sq(K, 0.0);
    parallel_for(K, threads, [&](int64_t k0, int64_t k1) {
      for (int64_t k = k0; k < k1; ++k) {
        double* row = &R[size_t(k) * N];
        for (int i = 0; i < r; ++i) {
          const double a = bf16_bits_to_f32(L->l1[size_t(k) * r + i]);
          const double* v = &l2d[size_t(i) * N];
          for (int64_t n = 0; n < N; ++n) row[n] = row[n] - a * v[n];
        }
        double sq = 0;
        for (int64_t n = 0; n < N; ++n) sq += row[n] * row[n];
        row_sq[k] = sq;
      }
    });
    {
      double s = 0;
      for (double v : row_sq) s += v;
      L->resid_bf16 = std::sqrt(s);
    }

    // 5. R^T as float32 [N, K] (uninitialised, then written whole; tiled as
    //    in step 2) and its largest magnitude, then the tensor scale and the
    //    NVFP4 codes into the image
    std::unique_ptr<float[]> rt_buf(new float[size_t(N) * K]);
    float* rt = rt_buf.get();
    std::vector<float> tile_max(ceil_div(N, 64), 0.0f);
    parallel_for(ceil_div(N, 64), threads, [&](int64_t b0, int64_t b1) {
      float tile[64][64];
      for (int64_t nb = b0 * 64; nb < std::min(N, b1 * 64); nb += 64) {
        const int64_t nn = std::min<int64_t>(64, N - nb);
        float m = 0.0f;
        for (int64_t kb = 0; kb < K; kb += 64) {
          const int64_t kn = std::min<int64_t>(64, K - kb);
          for (int64_t i = 0; i < kn; ++i) {
            const double* row = R + size_t(kb + i) * N + nb;
            for (int64_t j = 0; j < nn; ++j) tile[j][i] = float(row[j]);
          }
          for (int64_t j = 0; j < nn; ++j) {
            float* out = rt + size_t(nb + j) * K + kb;
            for (int64_t i = 0; i < kn; ++i) {
              out[i] = tile[j][i];
              m = std::max(m, std::fabs(tile[j][i]));
            }
          }
        }
        tile_max[nb / 64] = m;
      }
    });
    if (d->flags & SVDQ_PREPARE_KEEP_R) {
      L->r32.resize(size_t(K) * N);
      parallel_for(K, threads, [&](int64_t k0, int64_t k1) {
        for (int64_t k = k0; k < k1; ++k)
          for (int64_t n = 0; n < N; ++n) L->r32[size_t(k) * N + n] = float(R[size_t(k) * N + n]);
      });
    }
    r_buf.reset();
    const bool int4 = d->format == SVDQ_FMT_INT4;
    float amax_r = 0.0f;
    for (float v : tile_max) amax_r = std::max(amax_r, v);
    L->g_w = global_scale(amax_r);
    const float c_w = 1.0f / (6.0f * L->g_w);

    // static activation tensor scale from the calibration maxima:
    // max_j bf16(a_j / lambda_j) equals max|X_hat| of the calibration rows
    float amax_xh = 0.0f;
    for (int64_t k = 0; k < K; ++k)
      amax_xh = std::max(amax_xh, bf16_bits_to_f32(f32_to_bf16_bits(d->act_amax[k] * L->inv_lam[k])));
    L->g_a = global_scale(amax_xh);
    L->c_a = 1.0f / (6.0f * L->g_a);
    L->alpha = L->g_a * L->g_w;
    L->inv_alpha = 1.0f / L->alpha;

    // 6. the device image
    L->image.assign(g.total, 0);
    uint8_t* img = L->image.data();
    float* lam_img = reinterpret_cast<float*>(img + g.off_lam);
    float* inv_img = reinterpret_cast<float*>(img + g.off_inv_lam);
    for (int64_t k = 0; k < g.KC * kKChunk; ++k) {
      lam_img[k] = k < K ? L->lam[k] : 1.0f;
      inv_img[k] = k < K ? L->inv_lam[k] : 1.0f;
    }
    if (d->bias) std::memcpy(img + g.off_bias, d->bias, sizeof(uint16_t) * N);
    if (!int4) {
      parallel_for(N, threads, [&](int64_t n0, int64_t n1) {
        for (int64_t n = n0; n < n1; ++n)
          quantize_row(rt + size_t(n) * K, K, L->g_w, c_w,
                       [&](int64_t k, uint8_t byte) { img[bcode_off(g, n, k)] = byte; },
                       [&](int64_t s, uint8_t code) { img[bsf_off(g, n, s)] = code; });
      });
    } else {
      // INT4 codes and bf16 group scales of R^T, then the power-of-two prescales that keep
      // the kernel's f16 operands q s 2^e in range: the weights' largest value at most 2^15,
      // the calibration maximum of the activations at most 2^11 (headroom for inputs above it)
      std::vector<float> row_smax(N, 0.0f);
      parallel_for(N, threads, [&](int64_t n0, int64_t n1) {
        for (int64_t n = n0; n < n1; ++n)
          row_smax[n] = quantize_row_int4(
              rt + size_t(n) * K, K, [&](int64_t k, uint8_t byte) { img[int4_bcode_off(g, n, k)] = byte; },
              [&](int64_t c, uint16_t sb) { std::memcpy(img + int4_bsf_off(g, n, c), &sb, 2); });
      });
      float smax = 0.0f;
      for (float v : row_smax) smax = std::max(smax, v);
      const int ew = pow2_exponent(7.0 * double(smax), 15);
      const int ea = pow2_exponent(double(amax_xh), 11);
      L->g_w = std::ldexp(1.0f, -ew);
      L->g_a = std::ldexp(1.0f, -ea);
      L->c_a = 0.0f;
      L->alpha = std::ldexp(1.0f, -(ea + ew));
      L->inv_alpha = std::ldexp(1.0f, ea + ew);
    }
    for (int64_t k = 0; k < K; ++k)
      for (int i = 0; i < r; ++i) {
        const uint16_t v = L->l1[size_t(k) * r + i];
        std::memcpy(img + l1t_off(g, i, k), &v, 2);
      }
    for (int i = 0; i < r; ++i)
      for (int64_t n = 0; n < N; ++n) {
        const uint16_t v = L->l2[size_t(i) * N + n];
        std::memcpy(img + l2t_off(g, n, i), &v, 2);
      }
  } catch (const std::bad_alloc&) {
    return *err = "host allocation failed during preparation", SVDQ_ERR_HOST_ALLOC;
  } catch (const std::exception& e) {
    return *err = std::string("preparation failed: ") + e.what(), SVDQ_ERR_INTERNAL;
  }
  *out = L.release();
  return SVDQ_OK;
}

// ---------------------------------------------------------------- exports

// W4A16: W' = f32(W diag(s)) quantized row by row with the same NVFP4 quantizer
// as the W4A4 residual, under the tensor scale g = max|W'| / 2688.
svdq_status w4a16_quantize(const svdq_w4a16_desc* d, std::vector<uint8_t>* image, std::vector<uint8_t>* codes,
                           std::vector<uint8_t>* scales, float* g_out, std::string* err) {
  if (!d || !d->W) {
    *err = "descriptor and W are required";
    return SVDQ_ERR_INVALID_ARGUMENT;
  }
  const int64_t K = d->K, N = d->N;
  if (K < 64 || K % 64 || K > 12288 || N < 1 || N > (int64_t(1) << 24)) {
    *err = "K must be a multiple of 64 in [64, 12288] and N in [1, 2^24]";
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  }
  std::vector<float> s(size_t(K), 1.0f);
  if (d->s)
    for (int64_t k = 0; k < K; ++k) {
      s[size_t(k)] = d->s[k];
      if (!(s[size_t(k)] > 0.0f) || !std::isfinite(s[size_t(k)])) {
        *err = "s must be positive and finite";
        return SVDQ_ERR_INVALID_ARGUMENT;
      }
    }
  // two passes over W' = f32(W diag(s)), one row at a time (no N x K copy): its maximum, then the codes
  const uint16_t* W = static_cast<const uint16_t*>(d->W);
  const int threads = int(std::max(1u, std::min(16u, std::thread::hardware_concurrency())));
  auto scaled_row = [&](int64_t n, float* out) {
    for (int64_t k = 0; k < K; ++k) out[k] = bf16_bits_to_f32(W[size_t(n) * K + k]) * s[size_t(k)];
  };
  std::vector<float> part_max(size_t(threads), 0.0f);
  {
    std::atomic<int> next_slot{0};
    parallel_for(N, threads, [&](int64_t n0, int64_t n1) {
      const int slot = next_slot.fetch_add(1);
      std::vector<float> row(static_cast<size_t>(K));
      float m = 0.0f;
      for (int64_t n = n0; n < n1; ++n) {
        scaled_row(n, row.data());
        for (int64_t k = 0; k < K; ++k) m = std::max(m, std::fabs(row[size_t(k)]));
      }
      part_max[size_t(slot)] = m;
    });
  }
  float amax = 0.0f;
  for (float m : part_max) amax = std::max(amax, m);  // max is order-independent: exact
  const float g = global_scale(amax);
  const float c = 1.0f / (6.0f * g);
  codes->assign(size_t(N) * size_t(K / 2), 0);
  scales->assign(size_t(N) * size_t(K / 16), 0);
  uint8_t* cr = codes->data();
  uint8_t* sr = scales->data();
  parallel_for(N, threads, [&](int64_t n0, int64_t n1) {
    std::vector<float> row(static_cast<size_t>(K));
    for (int64_t n = n0; n < n1; ++n) {
      scaled_row(n, row.data());
      quantize_row(row.data(), K, g, c,
                   [&](int64_t k, uint8_t byte) { cr[size_t(n) * size_t(K / 2) + size_t(k / 2)] = byte; },
                   [&](int64_t sb, uint8_t code) { sr[size_t(n) * size_t(K / 16) + size_t(sb)] = code; });
    }
  });
  // the device image: tiles of 16 rows x 64 inputs in fragment order
  const W4A16Geom geo = make_w4a16_geom(K, N);
  image->assign(geo.total, 0);
  uint8_t* img = image->data();
  float* inv = reinterpret_cast<float*>(img + geo.off_inv_s);
  for (int64_t k = 0; k < K; ++k) inv[k] = 1.0f / s[size_t(k)];
  if (d->bias) std::memcpy(img + geo.off_bias, d->bias, sizeof(uint16_t) * size_t(N));
  for (int64_t nt = 0; nt < geo.N16 / 16; ++nt)
    for (int64_t kt = 0; kt < geo.KT; ++kt) {
      uint8_t* ct = img + geo.off_codes + size_t(nt * geo.KT + kt) * 512;
      uint8_t* st = img + geo.off_scales + size_t(nt * geo.KT + kt) * 64;
      for (int t = 0; t < 32; ++t)
        for (int j = 0; j < 4; ++j)
          for (int q = 0; q < 4; ++q) {
            const int64_t row = nt * 16 + (t >> 2) + 8 * (q & 1);
            const int64_t k = kt * 64 + 16 * j + 2 * (t & 3) + 8 * (q >> 1);
            ct[t * 16 + j * 4 + q] = row < N ? cr[size_t(row) * size_t(K / 2) + size_t(k / 2)] : 0;
          }
      for (int gi = 0; gi < 8; ++gi)
        for (int h = 0; h < 2; ++h)
          for (int j = 0; j < 4; ++j) {
            const int64_t row = nt * 16 + gi + 8 * h;
            st[gi * 8 + h * 4 + j] = row < N ? sr[size_t(row) * size_t(K / 16) + size_t(kt * 4 + j)] : 0;
          }
    }
  *g_out = g;
  return SVDQ_OK;
}

svdq_status export_array(const svdq_layer* L, int what, void* dst, size_t bytes, std::string* err) {
  const LayerGeom& g = L->g;
  const int64_t K = g.K, N = g.N, r = g.rank;
  auto need = [&](size_t n) -> svdq_status {
    if (bytes < n) {
      *err = "export buffer too small: need " + std::to_string(n) + " bytes";
      return SVDQ_ERR_BUFFER_TOO_SMALL;
    }
    return SVDQ_OK;
  };
  svdq_status st;
  uint8_t* out = static_cast<uint8_t*>(dst);
  switch (what) {
    case SVDQ_EXPORT_LAMBDA:
      if ((st = need(K * 4))) return st;
      std::memcpy(out, L->lam.data(), K * 4);
      return SVDQ_OK;
    case SVDQ_EXPORT_INV_LAMBDA:
      if ((st = need(K * 4))) return st;
      std::memcpy(out, L->inv_lam.data(), K * 4);
      return SVDQ_OK;
    case SVDQ_EXPORT_L1:
      if ((st = need(K * r * 2))) return st;
      std::memcpy(out, L->l1.data(), K * r * 2);
      return SVDQ_OK;
    case SVDQ_EXPORT_L2:
      if ((st = need(r * N * 2))) return st;
      std::memcpy(out, L->l2.data(), r * N * 2);
      return SVDQ_OK;
    case SVDQ_EXPORT_R:
      if (L->r32.empty()) return *err = "R was not kept (prepare with SVDQ_PREPARE_KEEP_R)", SVDQ_ERR_INVALID_ARGUMENT;
      if ((st = need(K * N * 4))) return st;
      std::memcpy(out, L->r32.data(), K * N * 4);
      return SVDQ_OK;
    case SVDQ_EXPORT_W_CODES:
      if ((st = need(N * K / 2))) return st;
      for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; k += 2)
          out[n * (K / 2) + k / 2] =
              L->image[L->format == SVDQ_FMT_INT4 ? int4_bcode_off(g, n, k) : bcode_off(g, n, k)];
      return SVDQ_OK;
    case SVDQ_EXPORT_W_SCALES:
      if (L->format == SVDQ_FMT_INT4) {  // bf16 bits [N, K / 64]
        if ((st = need(N * (K / 64) * 2))) return st;
        for (int64_t n = 0; n < N; ++n)
          for (int64_t c = 0; c < K / 64; ++c) std::memcpy(out + (n * (K / 64) + c) * 2, &L->image[int4_bsf_off(g, n, c)], 2);
        return SVDQ_OK;
      }
      if ((st = need(N * K / 16))) return st;
      for (int64_t n = 0; n < N; ++n)
        for (int64_t s = 0; s < K / 16; ++s) out[n * (K / 16) + s] = L->image[bsf_off(g, n, s)];
      return SVDQ_OK;
    case SVDQ_EXPORT_SIGMA:
      if (L->sigma.empty()) return *err = "no singular values (rank 0 or caller factors)", SVDQ_ERR_INVALID_ARGUMENT;
      if ((st = need(r * 8))) return st;
      std::memcpy(out, L->sigma.data(), r * 8);
      return SVDQ_OK;
    case SVDQ_EXPORT_SCALARS: {
      if ((st = need(16))) return st;
      const float v[4] = {L->g_a, L->g_w, L->alpha, L->inv_alpha};
      std::memcpy(out, v, 16);
      return SVDQ_OK;
    }
    case SVDQ_EXPORT_RESID_NORM: {
      if ((st = need(16))) return st;
      const double v[2] = {L->resid_f64, L->resid_bf16};
      std::memcpy(out, v, 16);
      return SVDQ_OK;
    }
    default:
      *err = "unknown export id " + std::to_string(what);
      return SVDQ_ERR_INVALID_ARGUMENT;
  }
}

svdq_status act_unpack(const svdq_layer* L, int64_t M, const uint8_t* act, size_t bytes, uint8_t* codes,
                       uint8_t* scales, uint16_t* lr, std::string* err) {
  const LayerGeom& g = L->g;
  const ActGeom a = make_act_geom(g, M);
  if (bytes < a.total) {
    *err = "activation buffer copy too small: need " + std::to_string(a.total) + " bytes";
    return SVDQ_ERR_BUFFER_TOO_SMALL;
  }
  const int64_t K = g.K;
  const bool int4 = L->format == SVDQ_FMT_INT4;
  for (int64_t m = 0; m < M; ++m) {
    if (codes)
      for (int64_t k = 0; k < K; k += 2)
        codes[m * (K / 2) + k / 2] = act[int4 ? int4_acode_off(a, m, k) : acode_off(a, m, k)];
    if (scales && int4)  // bf16 bits [M, K / 64]
      for (int64_t c = 0; c < K / 64; ++c) std::memcpy(scales + (m * (K / 64) + c) * 2, act + int4_asf_off(a, m, c), 2);
    else if (scales)
      for (int64_t s = 0; s < K / 16; ++s) scales[m * (K / 16) + s] = act[asf_off(a, m, s)];
    if (lr)
      for (int64_t rho = 0; rho < L->r_tot; ++rho) std::memcpy(&lr[m * L->r_tot + rho], act + lr_off(a, m, rho), 2);
  }
  return SVDQ_OK;
}

}  // namespace svdq
