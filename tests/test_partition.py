"""The tensor-core attention's tile partition (share_begin / share_of_tile in
csrc/common.cuh), compiled from the library's own header for the host and
checked on CPU: the ranges tile [0, T) in order, the first T % g CTAs take one
tile more, share_of_tile inverts share_begin, and "tile t starts the range of
the CTA that holds it" (the merge kernel's rule for which partial slots hold
a segment) marks exactly the first tile of every non-empty range."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

PROGRAM = r"""
#include <cstdio>
#include "common.cuh"
using salsc::share_begin;
using salsc::share_of_tile;
int main() {
  unsigned long long x = 88172645463325252ull;  // xorshift64
  auto rnd = [&](long long n) { x ^= x << 13; x ^= x >> 7; x ^= x << 17; return (long long)(x % n); };
  for (int trial = 0; trial < 4000; ++trial) {
    const long long g = 1 + rnd(300), T = 1 + rnd(trial % 2 ? 2000 : 600);
    const long long q = T / g, rem = T % g;
    if (share_begin(0, T, g) != 0 || share_begin(g, T, g) != T) return 1;
    long long starts = 0;
    for (long long c = 0; c < g; ++c) {
      const long long a = share_begin(c, T, g), b = share_begin(c + 1, T, g);
      if (b - a != (c < rem ? q + 1 : q)) return 2;
      if (b > a) ++starts;
    }
    long long marked = 0;
    for (long long t = 0; t < T; ++t) {
      const long long c = share_of_tile(t, T, g);
      if (c < 0 || c >= g || t < share_begin(c, T, g) || t >= share_begin(c + 1, T, g)) return 3;
      marked += share_begin(c, T, g) == t;
    }
    if (marked != starts) return 4;
  }
  std::printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(not os.path.exists(NVCC), reason="nvcc not found")
def test_tile_partition_host_build(tmp_path):
    src = tmp_path / "partition.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "partition"
    subprocess.run([NVCC, "-std=c++17", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "latent_space_sparse_b200", "csrc"),
                    str(src), "-o", str(exe)], check=True, capture_output=True, timeout=300)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
