// parallel.h -- the fixed-partition parallel loop of the host preparation.
#pragma once

#include <algorithm>
#include <cstdint>
#include <exception>
#include <thread>
#include <vector>

namespace svdq {

// f(begin, end) over [0, n) in at most `threads` contiguous pieces of
// ceil(n / threads) items (the last one shorter).  Each output of the loops
// that use it is computed inside one piece in a fixed order, so results do not
// depend on the thread count.
//
// Nothing here ends the process: a piece whose thread cannot be started runs
// on the calling thread, every started thread is joined, and the first
// exception a piece throws (std::bad_alloc, say) is rethrown to the caller
// after all pieces have stopped.
template <class F>
void parallel_for(int64_t n, int threads, F&& f) {
  if (threads <= 1 || n < 2) {
    f(int64_t(0), n);
    return;
  }
  const int64_t per = (n + threads - 1) / threads;
  std::vector<std::exception_ptr> errors(size_t(threads) + 1);
  std::vector<std::thread> pool;
  int64_t b = 0;
  int t = 0;
  try {
    pool.reserve(size_t(threads));
    for (; t < threads && b < n; ++t, b += per) {
      const int64_t e = std::min(n, b + per);
      std::exception_ptr* slot = &errors[size_t(t)];
      pool.emplace_back([&f, slot, b, e] {
        try {
          f(b, e);
        } catch (...) {
          *slot = std::current_exception();
        }
      });
    }
  } catch (...) {
    // no more threads: the pieces from b on run here
  }
  for (; b < n && !errors[size_t(threads)]; b += per) {
    try {
      f(b, std::min(n, b + per));
    } catch (...) {
      errors[size_t(threads)] = std::current_exception();
    }
  }
  for (auto& th : pool) th.join();
  for (auto& e : errors)
    if (e) std::rethrow_exception(e);
}

}  // namespace svdq
