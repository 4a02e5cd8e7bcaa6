"""The multiply-high divisors of the tile-block path (FastDiv in
csrc/internal.h): for every divisor d below 5,000 and a few large ones, and
every n with n * d < 2^32 drawn from the edges and at random, the kernel's
formula umulhi(n, m) + (n & one) equals n / d.  Compiled on the host against
the library's own header, with the device helper restated as the same
arithmetic on 64-bit integers."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include <random>
#include <vector>
#include "internal.h"
int main() {
  std::vector<uint32_t> divisors;
  for (uint32_t d = 1; d < 5000; ++d) divisors.push_back(d);
  for (uint32_t d : {65535u, 100003u, 1048583u}) divisors.push_back(d);
  std::mt19937_64 rng(1);
  long long checked = 0;
  for (const uint32_t d : divisors) {
    const salad::FastDiv f = salad::make_fastdiv(d);
    const uint64_t lim = ((uint64_t)1 << 32) / d;  // the n with n * d < 2^32
    for (int k = 0; k < 400; ++k) {
      const uint64_t n = k < 200 ? (uint64_t)k % lim : (k < 220 ? lim - 1 - (k - 200) % lim : rng() % lim);
      const uint32_t q = (uint32_t)(((uint64_t)(uint32_t)n * f.m) >> 32) + ((uint32_t)n & f.one);
      if (q != (uint32_t)n / d) {
        std::printf("FAIL d=%u n=%llu\n", d, (unsigned long long)n);
        return 1;
      }
      ++checked;
    }
  }
  std::printf("ok %lld\n", checked);
  return 0;
}
"""


def test_fastdiv_is_exact(tmp_path):
    src = tmp_path / "fd.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "fd"
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-I/usr/local/cuda/include",
                           f"-I{os.path.join(ROOT, 'sparse_linear_hybrid_b200', 'csrc')}", str(src), "-o", str(exe)])
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and res.stdout.startswith("ok"), res.stdout
