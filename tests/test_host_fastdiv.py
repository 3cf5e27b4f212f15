"""The multiply-shift divider the kernels use for their unit decode and
stride counts (`FastDiv` in csrc/schedule.cuh, the round-up method: n / d =
(umulhi(n, m) + n) >> s for 0 <= n < 2^31), compiled for the host with g++
from the same header and held to plain integer division: every divisor up to
4096, powers of two and their neighbours up to 2^30, and divisors near 2^31,
at numerators from 0 to 2^31 - 1 (the edges around each multiple of the
divisor, the top of the range, and pseudo-random values)."""
import os
import shutil
import subprocess

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "differential_attention_swa_b200", "csrc")

PROGRAM = r"""
#include "schedule.cuh"
#include <cstdint>
#include <cstdio>
#include <vector>

int main() {
  unsigned long long checked = 0, bad = 0;
  unsigned long long x = 88172645463325252ull;  // xorshift64
  auto rnd = [&]() { x ^= x << 13; x ^= x >> 7; x ^= x << 17; return x; };
  std::vector<long long> ds;
  for (long long d = 1; d <= 4096; ++d) ds.push_back(d);
  for (int k = 12; k <= 30; ++k)
    for (long long e = -1; e <= 1; ++e) ds.push_back((1ll << k) + e);
  for (long long d : {3000017ll, 123456789ll, 1000000007ll, 2147483646ll, 2147483647ll}) ds.push_back(d);
  const long long top = 2147483647ll;
  for (long long d : ds) {
    const swa::FastDiv f = swa::make_fastdiv((int)d);
    auto check = [&](long long n) {
      if (n < 0 || n > top) return;
      ++checked;
      const int got = f((int)n);
      if (got != (int)(n / d)) {
        if (bad < 5) std::printf("d=%lld n=%lld got %d want %lld\n", d, n, got, n / d);
        ++bad;
      }
    };
    for (long long n : {0ll, 1ll, d - 1, d, d + 1, 2 * d - 1, 2 * d, top, top - 1, top / d * d, top / d * d - 1})
      check(n);
    for (int r = 0; r < 400; ++r) {
      const long long n = (long long)(rnd() % (unsigned long long)(top + 1));
      check(n);
      check(n / d * d);
      check(n / d * d - 1);
    }
  }
  std::printf("%llu %llu\n", checked, bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_fastdiv_matches_integer_division(tmp_path):
    src = tmp_path / "fastdiv.cpp"
    exe = tmp_path / "fastdiv"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)], check=True,
                   capture_output=True, text=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    checked, bad = (int(v) for v in run.stdout.split()[-2:])
    assert run.returncode == 0 and bad == 0, run.stdout
    assert checked > 4_000_000
