"""Host-side logic of the CUDA library that needs no GPU: the multiply-shift division the
kernels use to decode a tile index into (sample, window, head).  The test compiles a small
host program against the library's own header and checks it against exact integer division."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "swin3d_window_attention_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include <random>
#include "s3w_common.cuh"
int main() {
  std::mt19937_64 rng(12345);
  long long checked = 0, bad = 0;
  auto check = [&](uint32_t d, int n) {
    const s3w::FastDiv f = s3w::make_fastdiv(d);
    ++checked;
    if (s3w::fdiv(n, f) != n / static_cast<int>(d)) {
      if (bad < 5) std::printf("mismatch n=%d d=%u got %d\n", n, d, s3w::fdiv(n, f));
      ++bad;
    }
  };
  std::vector<uint32_t> divisors;
  for (uint32_t d = 1; d <= 4096; ++d) divisors.push_back(d);
  for (int i = 0; i < 2000; ++i) divisors.push_back(1u + static_cast<uint32_t>(rng() % 0x7fffffffu));
  for (uint32_t d : {1u << 20, (1u << 20) + 1, 0x7fffffffu, 0x40000000u, 0x40000001u})
    divisors.push_back(d);
  for (uint32_t d : divisors) {
    const int edges[] = {0, 1, static_cast<int>(d) - 1, static_cast<int>(d), 0x7fffffff, 0x7ffffffe};
    for (int n : edges)
      if (n >= 0) check(d, n);
    for (long long m : {2ll, 3ll, 1000ll}) {   // around multiples of d
      const long long base = m * d;
      for (long long n = base - 1; n <= base + 1; ++n)
        if (n >= 0 && n <= 0x7fffffff) check(d, static_cast<int>(n));
    }
    for (int i = 0; i < 200; ++i) check(d, static_cast<int>(rng() & 0x7fffffff));
  }
  std::printf("checked %lld bad %lld\n", checked, bad);
  return bad ? 1 : 0;
}
"""


def test_fast_division_matches_integer_division(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc) and shutil.which("nvcc") is None:
        pytest.skip("nvcc not available")
    src = tmp_path / "fastdiv.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "fastdiv"
    subprocess.run([nvcc, "-std=c++17", "-O2", "-I", CSRC, str(src), "-o", str(exe)], check=True,
                   capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "bad 0" in out.stdout
