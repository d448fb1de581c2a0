"""The masked attention's index logic, checked exhaustively on the CPU.

The tcgen05 kernel does not evaluate the HSTU-style mask key by key: each
unit walks the key blocks of `mask_key_range`, and each softmax row builds its
visibility words from the two intervals of `mask_row_intervals`.  Those
helpers are host-callable, so this test compiles a small host program against
the library's own header and compares, for every small user shape and mask
setting, (a) the interval words with the key-by-key predicate `mask_visible`,
(b) that predicate with the oracle's mask, and (c) that every visible key of
a query block lies inside the block's key range.  A second host program
checks the workspace layout (`make_layout`) over many batch shapes: every
region 256-byte aligned and disjoint, the no-alloc scratch and the per-call
clear ending where the kernels expect, the fused expert rows fitting.  No GPU
needed (nvcc only)."""
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


LAYOUT_HARNESS = r'''
#include <cstdio>
#include <vector>
#include <algorithm>
#include "common.cuh"
using namespace ptl;
// For each (T, U, dtype): print "OK" or the first broken invariant of the
// workspace layout.
int main() {
  long long T; int U, dt;
  while (scanf("%lld %d %d", &T, &U, &dt) == 3) {
    WsLayout L;
    if (!make_layout(T, U, dt ? PTL_BF16 : PTL_F32, &L)) { printf("REJECT\n"); continue; }
    const size_t es = dt ? 2 : 4;
    struct R { size_t off, bytes; const char* name; };
    std::vector<R> r = {
      {L.err, 4, "err"}, {L.items, 8 * (size_t)L.max_items, "items"}, {L.item_count, 4, "item_count"},
      {L.lvl_hist, 4 * (size_t)(L.max_levels + 1), "lvl_hist"}, {L.lvl_start, 4 * (size_t)(L.max_levels + 1), "lvl_start"},
      {L.lvl_fill, 4 * (size_t)(L.max_levels + 1), "lvl_fill"}, {L.ulist, 16 * (size_t)L.max_items * H, "ulist"},
      {L.uoff, 8 * ATT_MAX_CTAS, "uoff"}, {L.ucnt, 8 * ATT_MAX_CTAS, "ucnt"},
      {L.chunk_cnt, 4 * (size_t)L.n_chunks * E, "chunk_cnt"}, {L.lb, 4 * (32 + 32 * (size_t)L.n_gchunks), "lb"},
      {L.moe_done, 4 * (size_t)L.max_tiles * (MOE1_NT + MOE2_NT), "moe_done"},
      {L.xn, es * T * D, "xn"}, {L.qkv, es * T * QKV_N, "qkv"}, {L.attn, es * T * D, "attn"},
      {L.x1, 4 * T * D, "x1"}, {L.xn2, es * T * D, "xn2"}, {L.act0, es * T * D, "act0"}, {L.act1, es * T * D, "act1"},
      {L.idx, 4 * T * K, "idx"}, {L.wgt, 4 * T * K, "wgt"}, {L.perm, 8 * T, "perm"}, {L.pos, 8 * T, "pos"},
      {L.rowroute, 4 * (size_t)L.padded_rows, "rowroute"}, {L.tiles, 8 * (size_t)L.max_tiles, "tiles"},
      {L.route_meta, 128, "route_meta"}, {L.hbuf, es * (size_t)L.padded_rows * F, "hbuf"},
      {L.ybuf, dt ? 2 * (size_t)L.padded_rows * D : 4 * 2 * T * D, "ybuf"}, {L.head_p, 4 * T, "head_p"}};
    if (dt) r.push_back({L.xperm, 2 * (size_t)L.padded_rows * D, "xperm"});
    const char* bad = nullptr;
    for (auto& x : r) {
      if (x.off % 256 != 0) bad = x.name;
      if (x.off + x.bytes > L.total) bad = x.name;
    }
    std::sort(r.begin(), r.end(), [](const R& a, const R& b) { return a.off < b.off; });
    for (size_t i = 1; i < r.size(); ++i)
      if (r[i - 1].bytes && r[i - 1].off + r[i - 1].bytes > r[i].off) bad = r[i].name;
    // the no-alloc scratch holds [0, wl_end): the error word and the work list
    if (L.wl_end < L.ucnt + 8 * ATT_MAX_CTAS || L.wl_end > L.chunk_cnt) bad = "wl_end";
    // one memset per call clears [0, clear_end): up to the fused path's counters
    if (L.clear_end < L.moe_done + 4 * (size_t)L.max_tiles * (MOE1_NT + MOE2_NT) || L.clear_end > L.xn)
      bad = "clear_end";
    // the fused expert path puts expert e's rows at e * cap
    if ((int64_t)E * L.cap > L.padded_rows || L.cap < T || L.cap % MOE_BM) bad = "cap";
    // the no-alloc entry point's fixed array holds the scratch of every
    // batch within its stated limits
    if (T <= PTL_NOALLOC_MAX_TOKENS && U <= PTL_NOALLOC_MAX_USERS && L.wl_end > PTL_NOALLOC_SCRATCH_BYTES)
      bad = "noalloc";
    // work-list bound: every user's query blocks fit
    if (L.max_items < (T + ATT_BLK - 1) / ATT_BLK + std::min<long long>(U, T)) bad = "max_items";
    printf(bad ? "BAD %s\n" : "OK\n", bad);
  }
  return 0;
}
'''


def test_workspace_layout_invariants(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "layout.cu"
    src.write_text(LAYOUT_HARNESS)
    exe = tmp_path / "layout"
    subprocess.check_call([nvcc, "-std=c++17", "-O1", "-I", CSRC, "-o", str(exe), str(src)])
    shapes = [(T, U, dt) for T in (0, 1, 2, 127, 128, 129, 255, 256, 257, 1000, 6823, 6912, 44000, 65535, 65536, 65537, 1 << 20)
              for U in (1, 2, 60, 390, 4095, 4096, 4097) for dt in (0, 1)]
    inp = "\n".join(f"{T} {U} {dt}" for T, U, dt in shapes) + "\n"
    out = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True).stdout.split("\n")
    bad = [(s, o) for s, o in zip(shapes, out) if o != "OK"]
    assert not bad, bad[:5]

