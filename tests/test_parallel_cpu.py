"""The host preparation's parallel loop (csrc/parallel.h), compiled into a
small C++ driver: pieces cover [0, n) exactly once for any thread count, and
an exception thrown inside a piece (std::bad_alloc, say) reaches the caller
with its type, after every other piece has finished, instead of ending the
process."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_w4a4_quantized_b200", "csrc")

DRIVER = r"""
#include <atomic>
#include <cstdio>
#include <new>
#include <stdexcept>
#include <vector>
#include "parallel.h"

int main() {
  int bad = 0;
  for (int threads = 1; threads <= 9; ++threads)
    for (long n : {0L, 1L, 2L, 7L, 64L, 1000L}) {
      std::vector<std::atomic<int>> hits(size_t(n) + 1);
      svdq::parallel_for(n, threads, [&](int64_t b, int64_t e) {
        for (int64_t i = b; i < e; ++i) hits[size_t(i)]++;
      });
      for (long i = 0; i < n; ++i) bad += hits[size_t(i)] != 1;
    }
  // a piece that throws: the others still run to the end, the caller sees the exception
  for (int threads : {1, 3, 8}) {
    std::atomic<int> done{0};
    bool caught = false;
    try {
      svdq::parallel_for(80, threads, [&](int64_t b, int64_t e) {
        if (b == 0) throw std::bad_alloc();
        done += int(e - b);
      });
    } catch (const std::bad_alloc&) {
      caught = true;
    }
    const int per = (80 + threads - 1) / threads;
    bad += !caught;
    bad += threads > 1 && done != 80 - per;
    bad += threads == 1 && done != 0;
  }
  // several pieces throw: one exception reaches the caller
  try {
    svdq::parallel_for(100, 4, [&](int64_t, int64_t) { throw std::runtime_error("piece"); });
    bad += 1;
  } catch (const std::runtime_error&) {
  }
  std::printf("%d\n", bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_parallel_for_covers_once_and_propagates_exceptions(tmp_path):
    src = tmp_path / "driver.cpp"
    src.write_text(DRIVER)
    exe = tmp_path / "driver"
    subprocess.run(["g++", "-O1", "-std=c++17", "-pthread", "-I" + CSRC, str(src), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "0", (r.returncode, r.stdout, r.stderr)
