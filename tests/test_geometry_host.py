"""The chunk geometry of the verify kernels (csrc/geometry.h), compiled for
the host and checked exhaustively on small rows and at the largest ones, for
the streaming pass's and the resample pass's vectors per thread: the chunks
of a row cover every full vector exactly once and nothing past the row; the
units (u, warp) are in index order; the ragged end (fewer than one vector)
belongs to the last chunk; and no index overflows 32 bits at SPECDEC_MAX_V."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

DRIVER = r"""
#include "geometry.h"
#include <cstdio>
#include <vector>
#include <initializer_list>
using namespace specdec;
static long fails = 0, checks = 0;
static void row_case(int V, int vec, int up) {
  const int nv_full = V / vec;
  const int64_t cpr = chunks_per_row(nv_full, vec, up);
  const int CH = chunk_vecs(vec, up), UPT = chunk_upt(vec, up);
  if (UPT * kThreads != CH) ++fails;
  std::vector<int> seen(nv_full, 0);
  int total = 0;
  for (int sub = 0; sub < cpr; ++sub) {
    const int cnt = chunk_count(nv_full, sub, vec, up);
    if (cnt < 0 || cnt > CH) ++fails;
    if (sub < cpr - 1 && cnt != CH) ++fails;   // only the last chunk is short
    total += cnt;
    for (int u = 0; u < UPT; ++u)
      for (int w = 0; w < kThreads / 32; ++w)   // unit (u, w): 32 consecutive vectors
        for (int lane = 0; lane < 32; ++lane) {
          const int pos = stream_pos(u, w * 32 + lane);
          if (pos != (u * (kThreads / 32) + w) * 32 + lane) ++fails;  // unit order is index order
          if (pos < 0 || pos >= CH) ++fails;
          if (pos < cnt) { const int j = sub * CH + pos; if (j >= nv_full) ++fails; else ++seen[j]; }
        }
  }
  if (total != nv_full) ++fails;
  for (int j = 0; j < nv_full; ++j) { ++checks; if (seen[j] != 1) ++fails; }
  // the ragged end: fewer than one vector, one warp's lanes cover it
  const int tail = V - nv_full * vec;
  if (tail < 0 || tail >= vec + (vec == 1)) ++fails;
  if (tail > 32) ++fails;
}
int main() {
  for (int up : {kU, 4})
  for (int vec : {1, 4, 8}) {
    for (int V = 1; V <= 3 * chunk_vecs(vec, up) * vec + 20; V += (V < 300 ? 1 : 997)) row_case(V, vec, up);
    for (int V : {32000, 128256, 151936, 152064, 256000}) row_case(V, vec, up);
    // the largest row: every element index stays below 2^31
    const int64_t V = 1 << 24, nv_full = V / vec, cpr = chunks_per_row(nv_full, vec, up);
    const int64_t last = ((cpr - 1) * chunk_vecs(vec, up) + chunk_vecs(vec, up) - 1) * vec + vec;
    if (last >= (int64_t(1) << 31)) ++fails;
    if (cpr > 65535) ++fails;                      // fits a grid dimension
  }
  std::printf("%ld %ld\n", checks, fails);
  return fails != 0;
}
"""


def test_chunk_geometry(tmp_path):
    src = tmp_path / "geom.cpp"
    src.write_text(DRIVER)
    exe = tmp_path / "geom"
    inc = os.path.join(ROOT, "speculative_decoding_draft_decode_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O2", "-I", inc, str(src), "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    checks, fails = map(int, res.stdout.split())
    assert checks > 100000
    assert fails == 0 and res.returncode == 0
