// svd.h -- truncated SVD used by the host preparation (see svd.cpp).
#pragma once

#include <stdint.h>

#include <vector>

namespace svdq {

struct SvdFactors {
  int64_t K = 0, N = 0;
  int r = 0;
  std::vector<double> U;      // [K x r] row-major, orthonormal columns
  std::vector<double> sigma;  // [r] descending
  std::vector<double> Vt;     // [r x N] row-major, orthonormal rows
};

// Top-r singular triplets of A [K x N] (row-major, float64).
void randomized_svd(const double* A, int64_t K, int64_t N, int r, int oversample, int power_iters,
                    uint64_t seed, int threads, SvdFactors* out);

}  // namespace svdq
