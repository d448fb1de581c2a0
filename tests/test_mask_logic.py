"""The masked attention's index logic, checked exhaustively on the CPU.

The tcgen05 kernel does not evaluate the HSTU-style mask key by key: each
unit walks the key blocks of `mask_key_range`, and each softmax row builds its
visibility words from the two intervals of `mask_row_intervals`.  Those
helpers are host-callable, so this test compiles a small host program against
the library's own header and compares, for every small user shape and mask
setting, (a) the interval words with the key-by-key predicate `mask_visible`,
(b) that predicate with the oracle's mask, and (c) that every visible key of
a query block lies inside the block's key range.  No GPU needed (nvcc only)."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import ptl_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "packed_sequence_transformer_b200", "csrc")

HARNESS = r'''
#include <cstdio>
#include "common.cuh"
using namespace ptl;
// For one user shape and mask: print the L x L visibility from the interval
// words ('1'/'0' per key), then "ERR" lines for any disagreement with the
// key-by-key predicate or any visible key outside its block's key range.
int main(int argc, char** argv) {
  int L, causal, C, N, G, W;
  while (scanf("%d %d %d %d %d %d", &L, &causal, &C, &N, &G, &W) == 6) {
    AttnMask m{nullptr, nullptr, causal, G, W};
    const int Hs = L - N;
    printf("CASE %d %d %d %d %d %d\n", L, causal, C, N, G, W);
    for (int i = 0; i < L; ++i) {
      int a0, b0, a1, b1;
      mask_row_intervals(i, L, C, Hs, m, a0, b0, a1, b1);
      for (int j0 = 0; j0 < L; j0 += 32) {
        const unsigned bits = interval_bits32(a0, b0, j0) | interval_bits32(a1, b1, j0);
        for (int k = 0; k < 32 && j0 + k < L; ++k) {
          const bool vi = (bits >> k) & 1u;
          const bool vp = mask_visible(i, j0 + k, C, Hs, m);
          putchar(vi ? '1' : '0');
          if (vi != vp) printf("\nERR interval %d %d\n", i, j0 + k);
        }
      }
      putchar('\n');
    }
    for (int b = 0; b * ATT_BLK < L; ++b) {
      int lo, hi;
      mask_key_range(b, L, C, Hs, m, lo, hi);
      for (int i = b * ATT_BLK; i < L && i < (b + 1) * ATT_BLK; ++i)
        for (int j = 0; j < L; ++j)
          if (mask_visible(i, j, C, Hs, m) && (j < lo || j > hi)) printf("ERR range %d %d %d\n", b, i, j);
    }
  }
  return 0;
}
'''


def _cases():
    out = []
    for L in (1, 2, 5, 33, 130, 300):
        for causal in (1, 0):
            for C in sorted({0, 1, L // 3}):
                for N in sorted({0, 1, (L - C) // 2}):
                    for G in (1, 3):
                        for W in (0, 1, 7, 140):
                            if C + N <= L:
                                out.append((L, causal, C, N, G, W))
    return out


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("masklogic")
    src = d / "harness.cu"
    src.write_text(HARNESS)
    exe = d / "harness"
    subprocess.check_call([nvcc, "-std=c++17", "-O1", "-I", CSRC, "-o", str(exe), str(src)])
    return exe


def test_interval_words_predicate_and_key_ranges_agree_with_the_oracle(harness):
    cases = _cases()
    inp = "\n".join(" ".join(map(str, c)) for c in cases) + "\n"
    res = subprocess.run([str(harness)], input=inp, capture_output=True, text=True, check=True)
    lines = res.stdout.splitlines()
    errs = [ln for ln in lines if ln.startswith("ERR")]
    assert not errs, errs[:10]
    k = 0
    n_checked = 0
    for c in cases:
        assert lines[k] == "CASE " + " ".join(map(str, c))
        L, causal, C, N, G, W = c
        rows = lines[k + 1:k + 1 + L]
        k += 1 + L
        got = np.array([[ch == "1" for ch in r] for r in rows], dtype=bool)
        want = O.hstu_user_mask(L, bool(causal), C, N, G, W)
        assert np.array_equal(got, want), c
        n_checked += 1
    assert n_checked == len(cases) > 500
