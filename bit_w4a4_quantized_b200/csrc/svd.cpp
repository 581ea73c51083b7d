// svd.cpp -- truncated SVD of the smoothed weight for the low-rank branch.
//
// The SVDQuant summary page (section 4.2, "Absorb magnified weight outliers
// with a low-rank branch") keeps the top-r singular triplets of W_hat:
// L1 = U_r Sigma_r, L2 = V_r^T.  Only r << min(K, N) triplets are needed, so
// this uses randomized subspace iteration (Halko, Martinsson & Tropp 2011,
// "Finding structure with randomness", Alg. 4.4 with re-orthonormalization):
//   Y = A Omega; repeat q times { Q = orth(Y); Z = orth(A^T Q); Y = A Z };
//   Q = orth(Y); G = A^T Q (= B^T with B = Q^T A);
// then a one-sided Jacobi (Hestenes) SVD of the thin G = V Sigma J^T gives
// B = J Sigma V^T and A ~ (Q J) Sigma V^T.
//
// Every parallel loop has a fixed partition and a fixed reduction order, so
// the result depends only on the inputs and the seed, not on the thread count.
#include "svd.h"

#include "parallel.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <immintrin.h>
#include <numeric>
#include <thread>
#include <vector>

namespace svdq {

namespace {

// splitmix64 (Steele, Lea & Flood 2014) -> uniform doubles -> Box-Muller normals.
struct Rng {
  uint64_t s;
  uint64_t next() {
    uint64_t z = (s += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
  double uniform() { return (double(next() >> 11) + 0.5) * (1.0 / 9007199254740992.0); }
  void normals(double* out, size_t n) {
    const double two_pi = 6.283185307179586476925286766559;
    for (size_t i = 0; i < n; i += 2) {
      double u1 = uniform(), u2 = uniform();
      double rad = std::sqrt(-2.0 * std::log(u1));
      out[i] = rad * std::cos(two_pi * u2);
      if (i + 1 < n) out[i + 1] = rad * std::sin(two_pi * u2);
    }
  }
};

// out[i][c] = fma(M[i][j], V[j][c], out[i][c]) for j = 0 .. jn-1 in order, for
// rows i < rows and columns c < l (M row stride ldm, V and out row stride l).
// Every output is one chain of fused multiply-adds in ascending j, whatever
// the blocking, so callers may split j into consecutive blocks.  Tiles of
// 4 rows x 8 columns keep 8 accumulators in AVX2 registers.
void accumulate_rows(const double* M, int64_t ldm, int64_t rows, int64_t jn, const double* V, int l,
                     double* out) {
  const int l8 = l / 8 * 8;
  int64_t i = 0;
  for (; i + 4 <= rows; i += 4) {
    const double* m0 = M + i * ldm;
    const double* m1 = m0 + ldm;
    const double* m2 = m1 + ldm;
    const double* m3 = m2 + ldm;
    double* o = out + i * l;
    for (int c = 0; c < l8; c += 8) {
      __m256d a00 = _mm256_loadu_pd(o + c), a01 = _mm256_loadu_pd(o + c + 4);
      __m256d a10 = _mm256_loadu_pd(o + l + c), a11 = _mm256_loadu_pd(o + l + c + 4);
      __m256d a20 = _mm256_loadu_pd(o + 2 * l + c), a21 = _mm256_loadu_pd(o + 2 * l + c + 4);
      __m256d a30 = _mm256_loadu_pd(o + 3 * l + c), a31 = _mm256_loadu_pd(o + 3 * l + c + 4);
      const double* v = V + c;
      for (int64_t j = 0; j < jn; ++j, v += l) {
        const __m256d v0 = _mm256_loadu_pd(v), v1 = _mm256_loadu_pd(v + 4);
        __m256d b = _mm256_broadcast_sd(m0 + j);
        a00 = _mm256_fmadd_pd(b, v0, a00);
        a01 = _mm256_fmadd_pd(b, v1, a01);
        b = _mm256_broadcast_sd(m1 + j);
        a10 = _mm256_fmadd_pd(b, v0, a10);
        a11 = _mm256_fmadd_pd(b, v1, a11);
        b = _mm256_broadcast_sd(m2 + j);
        a20 = _mm256_fmadd_pd(b, v0, a20);
        a21 = _mm256_fmadd_pd(b, v1, a21);
        b = _mm256_broadcast_sd(m3 + j);
        a30 = _mm256_fmadd_pd(b, v0, a30);
        a31 = _mm256_fmadd_pd(b, v1, a31);
      }
      _mm256_storeu_pd(o + c, a00);
      _mm256_storeu_pd(o + c + 4, a01);
      _mm256_storeu_pd(o + l + c, a10);
      _mm256_storeu_pd(o + l + c + 4, a11);
      _mm256_storeu_pd(o + 2 * l + c, a20);
      _mm256_storeu_pd(o + 2 * l + c + 4, a21);
      _mm256_storeu_pd(o + 3 * l + c, a30);
      _mm256_storeu_pd(o + 3 * l + c + 4, a31);
    }
    for (int c = l8; c < l; ++c)
      for (int q = 0; q < 4; ++q) {
        const double* m = M + (i + q) * ldm;
        double acc = o[q * l + c];
        for (int64_t j = 0; j < jn; ++j) acc = std::fma(m[j], V[j * l + c], acc);
        o[q * l + c] = acc;
      }
  }
  for (; i < rows; ++i) {
    const double* m = M + i * ldm;
    double* o = out + i * l;
    for (int c = 0; c < l; ++c) {
      double acc = o[c];
      for (int64_t j = 0; j < jn; ++j) acc = std::fma(m[j], V[j * l + c], acc);
      o[c] = acc;
    }
  }
}

constexpr int64_t kBlockJ = 256;  // reduction block: 256 x l doubles of V stay in L2

// Y[K x l] = A[K x N] X[N x l], row-major.  Each thread owns a range of rows
// and walks N in blocks, reusing the block of X across its rows.
void mul_A_X(const double* A, int64_t K, int64_t N, const double* X, int l, double* Y, int threads) {
  parallel_for(K, threads, [&](int64_t k0, int64_t k1) {
    std::fill(Y + k0 * l, Y + k1 * l, 0.0);
    for (int64_t nb = 0; nb < N; nb += kBlockJ)
      accumulate_rows(A + k0 * N + nb, N, k1 - k0, std::min(kBlockJ, N - nb), X + nb * l, l, Y + k0 * l);
  });
}

// Z[N x l] = A^T Q, A [K x N], Q [K x l], row-major.  Each thread owns a
// range of rows of Z (columns of A) and walks K in blocks; a 64 x 256 panel of
// A^T is packed so that its rows are contiguous.
void mul_At_Q(const double* A, int64_t K, int64_t N, const double* Q, int l, double* Z, int threads) {
  parallel_for(N, threads, [&](int64_t n0, int64_t n1) {
    std::fill(Z + n0 * l, Z + n1 * l, 0.0);
    std::vector<double> panel(size_t(64) * kBlockJ);
    for (int64_t kb = 0; kb < K; kb += kBlockJ) {
      const int64_t kn = std::min(kBlockJ, K - kb);
      for (int64_t nt = n0; nt < n1; nt += 64) {
        const int64_t nn = std::min<int64_t>(64, n1 - nt);
        for (int64_t k0 = 0; k0 < kn; k0 += 8)  // in 8 x 8 sub-blocks: whole lines in, whole lines out
          for (int64_t j0 = 0; j0 < nn; j0 += 8) {
            const int64_t kc = std::min<int64_t>(8, kn - k0), jc = std::min<int64_t>(8, nn - j0);
            double t[8][8];
            for (int64_t a = 0; a < kc; ++a)
              for (int64_t b = 0; b < jc; ++b) t[a][b] = A[(kb + k0 + a) * N + nt + j0 + b];
            for (int64_t b = 0; b < jc; ++b)
              for (int64_t a = 0; a < kc; ++a) panel[size_t(j0 + b) * kBlockJ + k0 + a] = t[a][b];
          }
        accumulate_rows(panel.data(), kBlockJ, nn, kn, Q + kb * l, l, Z + nt * l);
      }
    }
  });
}

// Orthonormalize the l columns of a row-major [rows x l] matrix in place
// (modified Gram-Schmidt, two passes).  Columns that vanish are set to zero.
void orthonormalize(double* Y, int64_t rows, int l) {
  std::vector<double> col(size_t(rows) * l);  // column-major copy
  for (int64_t i = 0; i < rows; ++i)
    for (int c = 0; c < l; ++c) col[size_t(c) * rows + i] = Y[i * l + c];
  for (int c = 0; c < l; ++c) {
    double* v = &col[size_t(c) * rows];
    double norm0 = 0;
    for (int64_t i = 0; i < rows; ++i) norm0 += v[i] * v[i];
    norm0 = std::sqrt(norm0);
    for (int pass = 0; pass < 2; ++pass) {
      for (int p = 0; p < c; ++p) {
        const double* u = &col[size_t(p) * rows];
        double d = 0;
        for (int64_t i = 0; i < rows; ++i) d += u[i] * v[i];
        for (int64_t i = 0; i < rows; ++i) v[i] -= d * u[i];
      }
    }
    double norm = 0;
    for (int64_t i = 0; i < rows; ++i) norm += v[i] * v[i];
    norm = std::sqrt(norm);
    if (norm <= 1e-12 * norm0 || norm == 0.0) {
      std::fill(v, v + rows, 0.0);
    } else {
      for (int64_t i = 0; i < rows; ++i) v[i] /= norm;
    }
  }
  for (int64_t i = 0; i < rows; ++i)
    for (int c = 0; c < l; ++c) Y[i * l + c] = col[size_t(c) * rows + i];
}

// One-sided Jacobi on the columns of G (column-major, n rows x l cols, l even):
// G J = H with orthogonal columns; J (l x l, column-major) accumulates the
// rotations.  Round-robin pair ordering: each step rotates l/2 disjoint
// pairs, split across threads.
void jacobi_svd(std::vector<double>& G, int64_t n, int l, std::vector<double>& J, int threads) {
  J.assign(size_t(l) * l, 0.0);
  for (int i = 0; i < l; ++i) J[size_t(i) * l + i] = 1.0;
  std::vector<int> ring(l);
  std::iota(ring.begin(), ring.end(), 0);
  const double tol = 1e-15;
  for (int sweep = 0; sweep < 40; ++sweep) {
    for (int step = 0; step < l - 1; ++step) {
      parallel_for(l / 2, threads, [&](int64_t b, int64_t e) {
        for (int64_t pi = b; pi < e; ++pi) {
          int p = ring[pi], q = ring[l - 1 - pi];
          if (p > q) std::swap(p, q);
          double* gp = &G[size_t(p) * n];
          double* gq = &G[size_t(q) * n];
          double alpha = 0, beta = 0, gamma = 0;
          for (int64_t i = 0; i < n; ++i) {
            alpha += gp[i] * gp[i];
            beta += gq[i] * gq[i];
            gamma += gp[i] * gq[i];
          }
          if (gamma == 0.0 || std::fabs(gamma) <= tol * std::sqrt(alpha * beta)) continue;
          const double zeta = (beta - alpha) / (2.0 * gamma);
          const double t = (zeta >= 0 ? 1.0 : -1.0) / (std::fabs(zeta) + std::sqrt(1.0 + zeta * zeta));
          const double c = 1.0 / std::sqrt(1.0 + t * t), s = c * t;
          for (int64_t i = 0; i < n; ++i) {
            const double x = gp[i], y = gq[i];
            gp[i] = c * x - s * y;
            gq[i] = s * x + c * y;
          }
          double* jp = &J[size_t(p) * l];
          double* jq = &J[size_t(q) * l];
          for (int i = 0; i < l; ++i) {
            const double x = jp[i], y = jq[i];
            jp[i] = c * x - s * y;
            jq[i] = s * x + c * y;
          }
        }
      });
      // rotate the ring, keeping ring[0] fixed
      int last = ring[l - 1];
      for (int i = l - 1; i > 1; --i) ring[i] = ring[i - 1];
      ring[1] = last;
    }
    // convergence: check all pairs once more without rotating
    bool done = true;
    for (int p = 0; p < l && done; ++p)
      for (int q = p + 1; q < l && done; ++q) {
        const double* gp = &G[size_t(p) * n];
        const double* gq = &G[size_t(q) * n];
        double alpha = 0, beta = 0, gamma = 0;
        for (int64_t i = 0; i < n; ++i) {
          alpha += gp[i] * gp[i];
          beta += gq[i] * gq[i];
          gamma += gp[i] * gq[i];
        }
        if (gamma != 0.0 && std::fabs(gamma) > tol * std::sqrt(alpha * beta)) done = false;
      }
    if (done) break;
  }
}

}  // namespace

void randomized_svd(const double* A, int64_t K, int64_t N, int r, int oversample, int power_iters,
                    uint64_t seed, int threads, SvdFactors* out) {
  const int64_t mn = std::min(K, N);
  int l = int(std::min<int64_t>(r + oversample, mn));
  if (l % 2) ++l;  // even column count for the round-robin Jacobi ordering
  const bool pad_col = l > mn;
  const int lr = pad_col ? int(mn) : l;  // columns that carry data

  std::vector<double> omega(size_t(N) * l, 0.0);
  Rng rng{seed ^ 0x5344514Bull};
  {
    std::vector<double> g(size_t(N) * lr);
    rng.normals(g.data(), g.size());
    for (int64_t n = 0; n < N; ++n)
      for (int c = 0; c < lr; ++c) omega[size_t(n) * l + c] = g[size_t(n) * lr + c];
  }
  std::vector<double> Y(size_t(K) * l), Z(size_t(N) * l);
  mul_A_X(A, K, N, omega.data(), l, Y.data(), threads);
  orthonormalize(Y.data(), K, l);
  for (int it = 0; it < power_iters; ++it) {
    mul_At_Q(A, K, N, Y.data(), l, Z.data(), threads);
    orthonormalize(Z.data(), N, l);
    mul_A_X(A, K, N, Z.data(), l, Y.data(), threads);
    orthonormalize(Y.data(), K, l);
  }
  // G = A^T Q  [N x l] (row-major in Z), to column-major
  mul_At_Q(A, K, N, Y.data(), l, Z.data(), threads);
  std::vector<double> G(size_t(N) * l);
  for (int64_t n = 0; n < N; ++n)
    for (int c = 0; c < l; ++c) G[size_t(c) * N + n] = Z[size_t(n) * l + c];
  std::vector<double> J;
  jacobi_svd(G, N, l, J, threads);

  std::vector<double> sig(l);
  for (int c = 0; c < l; ++c) {
    double s = 0;
    for (int64_t n = 0; n < N; ++n) s += G[size_t(c) * N + n] * G[size_t(c) * N + n];
    sig[c] = std::sqrt(s);
  }
  std::vector<int> order(l);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return sig[a] > sig[b]; });

  out->K = K;
  out->N = N;
  out->r = r;
  out->sigma.assign(r, 0.0);
  out->U.assign(size_t(K) * r, 0.0);   // row-major K x r
  out->Vt.assign(size_t(r) * N, 0.0);  // row-major r x N
  for (int i = 0; i < r && i < l; ++i) {
    const int c = order[i];
    const double s = sig[c];
    out->sigma[i] = s;
    if (s > 0) {
      for (int64_t n = 0; n < N; ++n) out->Vt[size_t(i) * N + n] = G[size_t(c) * N + n] / s;
    }
    // U column i = Q * J[:, c]
    const double* jc = &J[size_t(c) * l];
    for (int64_t k = 0; k < K; ++k) {
      double acc = 0;
      const double* q = &Y[size_t(k) * l];
      for (int p = 0; p < l; ++p) acc += q[p] * jc[p];
      out->U[size_t(k) * r + i] = acc;
    }
  }
}

}  // namespace svdq
