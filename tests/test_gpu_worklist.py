"""The causal attention's unit lists, read back from the workspace after the
work-list kernel ran on the GPU.

The work list deals units (a 128-row query block of one user and one head,
walking b + 1 key blocks) heaviest first to the CTAs of the persistent grid
in snake order, each unit to the CTA's stream with fewer steps so far.  These
tests check, on seeded packings, that the (CTA, stream) lists cover every
(user, query block, head) exactly once, that they fit their array, that the
per-stream step counts add up to the causal total, and on the 60-user / 6823-
token packing that no stream walks more key blocks than its longest unit
needs (6) and no CTA more than 10.  The attention outputs themselves are
compared with the oracle in test_gpu_steps.py and test_gpu_layer.py."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "packed_sequence_transformer_b200", "csrc")
ATT_MAX_CTAS = 1024
H = 8

OFFSETS = r'''
#include <cstdio>
#include "common.cuh"
using namespace ptl;
int main() {
  long long T; int U;
  while (scanf("%lld %d", &T, &U) == 2) {
    WsLayout L;
    if (!make_layout(T, U, PTL_BF16, &L)) { printf("REJECT\n"); continue; }
    printf("%zu %zu %zu %lld\n", L.ulist, L.uoff, L.ucnt, (long long)L.max_items);
  }
  return 0;
}
'''


@pytest.fixture(scope="module")
def offsets_tool(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    d = tmp_path_factory.mktemp("wl")
    src = d / "offsets.cu"
    src.write_text(OFFSETS)
    exe = d / "offsets"
    subprocess.run([nvcc, "-std=c++17", "-I", CSRC, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)],
                   check=True, capture_output=True)

    def layout(T, U):
        out = subprocess.run([str(exe)], input=f"{T} {U}\n", capture_output=True, text=True, check=True).stdout
        ulist, uoff, ucnt, max_items = map(int, out.split())
        return ulist, uoff, ucnt, max_items
    return layout


def _lists(layout, lengths, seed):
    cu = S.offsets_from_lengths(lengths)
    T, U = int(cu[-1]), len(lengths)
    qkv = dev(np.random.default_rng(seed).standard_normal((T, 1536)).astype(np.float32), torch.bfloat16)
    ws = ptl.alloc_workspace(T, U, "bf16")
    out = torch.empty(T, 512, dtype=torch.bfloat16, device="cuda")
    ptl.attention(qkv, out, dev(cu, torch.int32), ws)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    ulist_off, uoff_off, ucnt_off, max_items = layout(T, U)
    raw = ws.view(torch.uint8).cpu().numpy()
    ucnt = raw[ucnt_off:ucnt_off + 8 * ATT_MAX_CTAS].view(np.int32)
    uoff = raw[uoff_off:uoff_off + 8 * ATT_MAX_CTAS].view(np.int32)
    ulist = raw[ulist_off:ulist_off + 16 * max_items * H].view(np.int32).reshape(-1, 4)
    G = min(max_items * H, torch.cuda.get_device_properties(0).multi_processor_count, ATT_MAX_CTAS)
    streams = [ulist[uoff[i]:uoff[i] + ucnt[i]] for i in range(2 * G)]
    return cu, streams


def _check_cover(cu, streams):
    """Every (user, block, head) exactly once.  Returns the per-stream
    key-block steps."""
    starts = {int(s): u for u, s in enumerate(cu[:-1]) if cu[u + 1] > cu[u]}
    seen = []
    loads = []
    for lst in streams:
        steps = 0
        for s0, L, b, h in lst:
            u = starts[int(s0)]
            assert L == cu[u + 1] - cu[u] and 0 <= b < (L + 127) // 128 and 0 <= h < H
            steps += b + 1
            seen.append((u, int(b), int(h)))
        loads.append(steps)
    want = {(u, b, h) for u in range(len(cu) - 1) for b in range((cu[u + 1] - cu[u] + 127) // 128) for h in range(H)}
    assert len(seen) == len(set(seen)) and set(seen) == want
    return np.array(loads)


def test_sixty_user_packing_lists(offsets_tool):
    cu, streams = _lists(offsets_tool, S.config1_lengths(), seed=41)
    loads = _check_cover(cu, streams)
    assert loads.sum() == 1064
    assert loads.max() == 6 and loads.reshape(-1, 2).sum(1).max() <= 10


@pytest.mark.parametrize("lengths", [
    [257, 600],
    [40, 257, 600, 12],
    [1, 127, 128, 129, 0, 300, 5, 513, 0],
    [1100, 3, 7, 700, 64],
    [4096] * 3 + [17] * 50,
    [1] * 300,
])
def test_lists_cover_every_unit_once(offsets_tool, lengths):
    cu, streams = _lists(offsets_tool, lengths, seed=42)
    loads = _check_cover(cu, streams)
    T, U = int(cu[-1]), len(lengths)
    assert sum(len(s) for s in streams) <= offsets_tool(T, U)[3] * H
    nb = [(L + 127) // 128 for L in lengths]
    assert loads.sum() == H * sum(n * (n + 1) // 2 for n in nb)
