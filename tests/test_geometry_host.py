"""The even split of the flattened row space over CTAs (csrc/geometry.h),
compiled for the host and checked exhaustively on small cases: the ranges
tile [0, T) without gaps or overlaps, every CTA gets floor(T/G) or
ceil(T/G) vectors, cta_of inverts the split, and slots_bound bounds the CTAs
meeting any row."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

DRIVER = r"""
#include "geometry.h"
#include <cstdio>
#include <initializer_list>
using namespace specdec;
int main() {
  long fails = 0, checks = 0;
  for (int64_t nv = 1; nv <= 40; ++nv)
  for (int64_t rows = 1; rows <= 30; ++rows) {
    const int64_t T = rows * nv;
    for (int64_t G = 1; G <= T && G <= 64; ++G) {
      int64_t prev_end = 0;
      for (int64_t c = 0; c < G; ++c) {
        int64_t b = part_begin(c, T, G), e = part_begin(c + 1, T, G);
        ++checks;
        if (b != prev_end) ++fails;
        if (e - b != T / G && e - b != (T + G - 1) / G) ++fails;
        for (int64_t v = b; v < e; ++v) if (cta_of(v, T, G) != c) ++fails;
        prev_end = e;
      }
      if (prev_end != T) ++fails;
      const int64_t bound = slots_bound(nv, T, G);
      for (int64_t r = 0; r < rows; ++r) {
        int64_t n = cta_of(r * nv + nv - 1, T, G) - cta_of(r * nv, T, G) + 1;
        if (n > bound) ++fails;
      }
      // a larger grid never needs fewer slots
      if (G > 1 && slots_bound(nv, T, G - 1) > bound) ++fails;
    }
  }
  // large values do not overflow
  const int64_t T = (int64_t)65536 * 33 * (1 << 21);
  for (int64_t G : {1, 148, 4096}) {
    if (part_begin(G, T, G) != T) ++fails;
    if (cta_of(T - 1, T, G) != G - 1) ++fails;
    if (cta_of(0, T, G) != 0) ++fails;
  }
  if (grid_upper(5000, 128, 4096) != 39 || grid_upper(10, 128, 4096) != 1 || grid_upper(1 << 30, 128, 1184) != 1184) ++fails;
  std::printf("%ld %ld\n", checks, fails);
  return fails != 0;
}
"""


def test_partition_properties(tmp_path):
    src = tmp_path / "geom.cpp"
    src.write_text(DRIVER)
    exe = tmp_path / "geom"
    inc = os.path.join(ROOT, "speculative_decoding_draft_decode_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", inc, str(src), "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True)
    checks, fails = map(int, res.stdout.split())
    assert checks > 10000
    assert fails == 0 and res.returncode == 0
