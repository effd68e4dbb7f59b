"""The kernel's division of row and token indices by a launch-invariant divisor
(multiply-high and shifts, DivU32 in fused_norm_kernel.cuh), compiled for the host and
checked against integer division: divisors of every bit length, the workloads' L and
tokens-per-frame values, and numerators at both ends of the 32-bit range and next to
multiples of the divisor. Host only (nvcc compiles, gcc-style host code runs)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rmsnorm_row_b200", "csrc")

SRC = r'''
#include "fused_norm_kernel.cuh"
#include <cstdio>
using namespace fused_norm_impl;
static uint64_t s = 0x9E3779B97F4A7C15ull;
static uint32_t rnd() { s ^= s << 13; s ^= s >> 7; s ^= s << 17; return (uint32_t)(s >> 16); }
static long bad = 0, n_checked = 0;
static void check(uint32_t n, uint32_t d, const DivU32& v) {
  ++n_checked;
  if (div_u32(n, v) != n / d) {
    if (bad < 5) std::printf("mismatch n=%u d=%u got=%u want=%u\n", n, d, div_u32(n, v), n / d);
    ++bad;
  }
}
int main() {
  const uint32_t fixed[] = {1u, 2u, 3u, 5u, 7u, 16u, 59u, 1237u, 3600u, 8400u, 90000u, 176400u,
                            65535u, 65536u, 65537u, 0x7FFFFFFFu, 0x80000000u, 0x80000001u, 0xFFFFFFFFu};
  for (int i = 0; i < 40 + 19; ++i) {
    uint32_t d;
    if (i < 19) d = fixed[i];
    else { int bits = 1 + (i - 19) % 32; d = (rnd() | 1u) >> (32 - bits); if (d == 0) d = 1; }
    const DivU32 v = make_div_u32(d);
    const uint32_t edges[] = {0u, 1u, d - 1u, d, d + 1u, 0xFFFFFFFFu, 0xFFFFFFFEu,
                              (0xFFFFFFFFu / d) * d, (0xFFFFFFFFu / d) * d - 1u, 0x80000000u};
    for (uint32_t n : edges) check(n, d, v);
    for (int k = 0; k < 60000; ++k) {
      const uint32_t n = rnd();
      check(n, d, v);
      const uint32_t m = (n / d) * d;  // next to a multiple of d
      check(m, d, v);
      if (m) check(m - 1u, d, v);
    }
  }
  std::printf("checked %ld mismatches %ld\n", n_checked, bad);
  return bad != 0;
}
'''


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_invariant_divisor_division_matches_integer_division(tmp_path):
    src = tmp_path / "fast_div.cu"
    src.write_text(SRC)
    exe = tmp_path / "fast_div"
    subprocess.run(["nvcc", "-O2", "-std=c++17", "--expt-relaxed-constexpr", "-I", CSRC,
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True, capture_output=True, timeout=600)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout
    assert "mismatches 0" in out.stdout
    assert int(out.stdout.split()[1]) > 10_000_000
