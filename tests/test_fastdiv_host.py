"""Division by a per-launch constant as multiply and shift (the grid helpers' FastDiv):
compiled from the library's own header for the host with nvcc and checked against integer
division -- every dividend below 2^17 for every divisor up to 4096, random and boundary
dividends up to 2^31 - 1, and large divisors.  No GPU needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_25_b200", "csrc")

PROGRAM = r'''
#include "bsa_kernels.cuh"
#include <cstdio>
int main() {
  unsigned long long bad = 0, checked = 0;
  unsigned long long x = 88172645463325252ull;
  auto check = [&](int n, int d, const bsa::FastDiv& f) {
    if (bsa::fdiv(n, f) != n / d) ++bad;
    ++checked;
  };
  for (int d = 1; d <= 4096; ++d) {
    const bsa::FastDiv f = bsa::make_fastdiv(d);
    for (int n = 0; n < (1 << 17); ++n) check(n, d, f);
    for (int k = 0; k < 512; ++k) {
      x ^= x << 13; x ^= x >> 7; x ^= x << 17;
      check(static_cast<int>(x & 0x7fffffffull), d, f);
    }
    const int edge[] = {0x7fffffff, 0x7ffffffe, d - 1, d, 2 * d - 1, 2 * d};
    for (int n : edge) check(n, d, f);
  }
  const int big[] = {0x7fffffff, 0x40000001, 0x40000000, 0x3fffffff, 65535, 65537, 92160};
  for (int d : big) {
    const bsa::FastDiv f = bsa::make_fastdiv(d);
    for (int k = 0; k < 200000; ++k) {
      x ^= x << 13; x ^= x >> 7; x ^= x << 17;
      check(static_cast<int>(x & 0x7fffffffull), d, f);
    }
    check(0x7fffffff, d, f);
    check(d - 1, d, f);
  }
  std::printf("%llu %llu\n", checked, bad);
  return bad != 0;
}
'''


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else shutil.which("nvcc")


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_fastdiv_matches_integer_division(tmp_path):
    src = tmp_path / "fastdiv_check.cu"
    exe = tmp_path / "fastdiv_check"
    src.write_text(PROGRAM)
    r = subprocess.run([_nvcc(), "-O2", "-std=c++17", "--expt-relaxed-constexpr", "-I", CSRC,
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    checked, bad = (int(v) for v in out.stdout.split())
    assert checked > 500_000_000
    assert bad == 0
