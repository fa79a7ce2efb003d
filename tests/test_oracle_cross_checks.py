"""The oracle against independent implementations and against planted
mistakes.

* Philox4x32-10: compared word for word with PyTorch's open-source Philox
  engine (ATen/core/PhiloxRNGEngine.h), compiled here from its header.
* Mutation checks: plausible mistakes are planted in a temporary copy of the
  oracle source (never in the oracle itself); each mutant must fail at least
  one of the pins in test_oracle_pins.py.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from oracle import build as oracle_build

import test_oracle_pins as pins
import test_oracle_adasd as adasd
import test_oracle_ngram as ngram

TORCH_PHILOX_MAIN = r"""
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>
int main() {
  unsigned c0, c1, c2, c3, k0, k1;
  while (std::scanf("%u %u %u %u %u %u", &c0, &c1, &c2, &c3, &k0, &k1) == 6) {
    uint64_t seed = ((uint64_t)k1 << 32) | k0;
    uint64_t subsequence = ((uint64_t)c3 << 32) | c2;
    at::Philox4_32 e(seed, subsequence, 0);
    e.set_offset(((uint64_t)c1 << 32) | c0);
    unsigned a = e(), b = e(), c = e(), d = e();
    std::printf("%u %u %u %u\n", a, b, c, d);
  }
}
"""


def test_philox_matches_pytorch_engine(tmp_path):
    import torch
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    src = tmp_path / "philox_main.cpp"
    src.write_text(TORCH_PHILOX_MAIN)
    exe = tmp_path / "philox_main"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", inc, str(src), "-o", str(exe)], check=True)
    rng = np.random.default_rng(123)
    cases = rng.integers(0, 2**32, size=(2000, 6), dtype=np.uint64)
    cases[:10] = 0
    cases[10:20] = 2**32 - 1
    text = "\n".join(" ".join(str(int(v)) for v in row) for row in cases) + "\n"
    res = subprocess.run([str(exe)], input=text, capture_output=True, text=True, check=True)
    got = np.array([[int(v) for v in ln.split()] for ln in res.stdout.strip().split("\n")], np.uint64)
    for row, want in zip(cases, got):
        mine = oracle.philox4x32_10(row[:4].astype(np.uint32), row[4:].astype(np.uint32))
        assert mine.tolist() == want.tolist()


# (name, original text, mutated text, pins that must catch it)
MUTANTS = [
    ("argmax ties to the highest index",
     "                      logit_at(logits, dtype, row_stride, row, best)) > 0)",
     "                      logit_at(logits, dtype, row_stride, row, best)) >= 0)",
     [lambda: pins.test_argmax_and_topk_match_sorting(7)]),
    ("draft compared with the next row's choice",
     "if (d[h] < 0 || d[h] >= V || d[h] != am[h]) break;",
     "if (d[h] < 0 || d[h] >= V || d[h] != am[h + 1]) break;",
     [pins.test_worked_example_greedy, pins.test_greedy_scan_brute_force]),
    ("bonus token taken from the previous row",
     "else if (i == h) out[i] = am[h];",
     "else if (i == h) out[i] = am[h > 0 ? h - 1 : 0];",
     [pins.test_worked_example_greedy, pins.test_all_accept_example]),
    ("scan does not stop at the first disagreement",
     "if (d[h] < 0 || d[h] >= V || d[h] != am[h]) break;  // first disagreement stops the scan\n        ++h;",
     "if (d[h] < 0 || d[h] >= V || d[h] != am[h]) { ++h; continue; }\n        ++h;",
     [pins.test_greedy_scan_brute_force]),
    ("NaN ranked above numbers",
     "    if (na) return -1;\n    if (nb) return 1;",
     "    if (na) return 1;\n    if (nb) return -1;",
     [lambda: pins.test_argmax_and_topk_match_sorting(33)]),
    ("residual with the wrong sign",
     "r[x] = std::max(0.0, p_of(h, x) - q_of(h, x));",
     "r[x] = std::max(0.0, q_of(h, x) - p_of(h, x));",
     [lambda: pins.test_rejection_preserves_target_distribution(8, 3, 1.0)]),
    ("accept test inverted (q/p instead of p/q)",
     "if (!(ua * qd < p)) break;",
     "if (!(ua * p < qd)) break;",
     [pins.test_rejection_expected_accept_len]),
    ("temperature multiplies instead of divides",
     "double sx = static_cast<double>(logit_at(target, dtype, row_stride, row0 + i, x)) / T;\n        return",
     "double sx = static_cast<double>(logit_at(target, dtype, row_stride, row0 + i, x)) * T;\n        return",
     [pins.test_rejection_softmax_closed_forms]),
    ("bonus sampled from row k-1",
     "for (int x = 0; x < V; ++x) { r[x] = p_of(k, x); S += r[x]; }",
     "for (int x = 0; x < V; ++x) { r[x] = p_of(k - 1, x); S += r[x]; }",
     [lambda: pins.test_rejection_preserves_target_distribution(8, 3, 1.0)]),
    ("Philox high words swapped",
     "uint32_t n0 = hi1 ^ c[1] ^ k[0];",
     "uint32_t n0 = hi0 ^ c[1] ^ k[0];",
     [pins.test_philox_known_answers]),
    ("tree: ties to the highest node index",
     "if (ok[c] && depth[c] > depth[best]) best = c;",
     "if (ok[c] && depth[c] >= depth[best]) best = c;",
     [pins.test_tree_brute_force_small]),
    ("tree: node matched against its own row",
     "ok[c] = ok[par[c]] && t >= 0 && t < V && t == am[par[c]];",
     "ok[c] = ok[par[c]] && t >= 0 && t < V && t == am[c];",
     [pins.test_tree_brute_force_small, pins.test_tree_chain_reduces_to_greedy]),
    ("n-gram: shortest suffix tried first",
     "for (int n = n_max; n >= n_min && !done; --n) {",
     "for (int n = n_min; n <= n_max && !done; ++n) {",
     [lambda: ngram.test_matches_literal_steps(0), ngram.test_known_answers]),
    ("n-gram: oldest occurrence instead of the most recent",
     "for (int j = L - n - 1; j >= 0 && !done; --j) {  // most recent first",
     "for (int j = 0; j <= L - n - 1 && !done; ++j) {  // most recent first",
     [lambda: ngram.test_matches_literal_steps(0), ngram.test_known_answers]),
    ("AdaSD: Jensen-Shannon mixture not halved",
     "const double m = 0.5 * (px + qx);",
     "const double m = (px + qx);",
     [lambda: adasd.test_matches_scipy(1.0), adasd.test_closed_forms]),
    ("AdaSD: divergence terms not halved",
     "if (px > 0.0) D += 0.5 * px * std::log(px / m);",
     "if (px > 0.0) D += px * std::log(px / m);",
     [lambda: adasd.test_matches_scipy(1.0), adasd.test_closed_forms]),
    ("AdaSD: entropy of the target instead of the draft",
     "if (qx > 0.0) H -= qx * std::log(qx);",
     "if (px > 0.0) H -= px * std::log(px);",
     [lambda: adasd.test_matches_scipy(1.0), adasd.test_closed_forms]),
    ("margin: sample distance not divided by S",
     "mg = std::min(mg, std::min(t - prev, c - t) / S);",
     "mg = std::min(mg, std::min(t - prev, c - t));",
     [pins.test_rejection_margin_sample_distance_over_S]),
    ("margin: accept test measured at the rejecting position only",
     "mg = std::min(mg, qd > 0.0 ? std::fabs(ua - p / qd) : p);\n        if (!(ua * qd < p)) break;",
     "if (!(ua * qd < p)) { mg = std::min(mg, qd > 0.0 ? std::fabs(ua - p / qd) : p); break; }",
     [pins.test_rejection_margin_accept_distance, pins.test_rejection_margin_zero_q_draft]),
    ("margin: residual mass S left out",
     "        mg = std::min(mg, S);\n",
     "",
     [pins.test_rejection_margin_residual_mass]),
]


def _build_mutant(tmp_path, idx, orig, new):
    src = open(oracle_build.SRC).read()
    assert src.count(orig) == 1, "mutation anchor not unique: %r" % orig
    path = tmp_path / ("mutant%d.cpp" % idx)
    path.write_text(src.replace(orig, new))
    so = tmp_path / ("mutant%d.so" % idx)
    subprocess.run(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", str(path), "-o", str(so)], check=True)
    return str(so)


@pytest.mark.parametrize("idx", range(len(MUTANTS)), ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, idx):
    name, orig, new, checks = MUTANTS[idx]
    so = _build_mutant(tmp_path, idx, orig, new)
    caught = False
    with oracle.use_library(so):
        for chk in checks:
            try:
                chk()
            except AssertionError:
                caught = True
                break
    assert caught, "planted mistake not caught: " + name
