"""Layer 0's LayerNorm1 as the layer path's prologue writes it, read back
from the workspace after one bf16 layer and compared, row by row for EVERY
row, with the oracle's LayerNorm (fp64) of the same bf16 input.

The prologue's row blocks take one wave (at most SMs - 2 blocks of 32 warps)
and each warp walks rows with a grid-wide stride, two rows' loads in flight:
the sizes below put the last row at the start, inside and at the end of a
stride, and past the second and third stride, so that a row the loop skips or
writes twice shows up (the workspace starts zeroed, and an unwritten row reads
as zeros).  Tolerance: the kernel's fp32 LayerNorm rounded to bf16 against the
fp64 oracle is within one bf16 unit in the last place, 2^-7 of the value, plus
1e-6 for values near zero."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import ptl
from packed_sequence_transformer_b200 import synthetic as S
from tests.gpu_util import dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "packed_sequence_transformer_b200", "csrc")
D = 512

OFFSETS = r'''
#include <cstdio>
#include "common.cuh"
using namespace ptl;
int main() {
  long long T; int U;
  while (scanf("%lld %d", &T, &U) == 2) {
    WsLayout L;
    if (!make_layout(T, U, PTL_BF16, &L)) { printf("REJECT\n"); continue; }
    printf("%zu\n", L.xn);
  }
  return 0;
}
'''


@pytest.fixture(scope="module")
def xn_offset(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    d = tmp_path_factory.mktemp("prologue")
    src = d / "offsets.cu"
    src.write_text(OFFSETS)
    exe = d / "offsets"
    subprocess.run([nvcc, "-std=c++17", "-I", CSRC, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)],
                   check=True, capture_output=True)

    def offset(T, U):
        out = subprocess.run([str(exe)], input=f"{T} {U}\n", capture_output=True, text=True, check=True).stdout
        return int(out.split()[0])
    return offset


def _rows_per_stride():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return 32 * max(1, sms - 2)


def _lengths(T):
    """T tokens as users of at most 700 tokens (a ragged last one)."""
    out = []
    while T > 0:
        out.append(min(700, T))
        T -= out[-1]
    return out


@pytest.mark.parametrize("which", ["one", "few", "stride", "stride+1", "two+1", "three+17"])
def test_prologue_layernorm_rows(xn_offset, which):
    W = _rows_per_stride()
    T = {"one": 1, "few": 37, "stride": W, "stride+1": W + 1, "two+1": 2 * W + 1, "three+17": 3 * W + 17}[which]
    lengths = _lengths(T)
    c = S.make_case("prologue", lengths=lengths, seed=71, dtype="bf16", num_layers=1)
    assert c.total_tokens == T
    x_bf = O.round_bf16(c.x)
    x = dev(c.x, torch.bfloat16)
    out = torch.empty_like(x)
    cu = dev(c.cu_seqlens, torch.int32)
    ws = ptl.alloc_workspace(T, len(lengths), "bf16")
    ptl.layer_forward(x, out, cu, ptl.to_device_layer(c.layers[0], "bf16"), ws)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    off = xn_offset(T, len(lengths))
    raw = ws.view(torch.uint8)[off:off + T * D * 2].cpu()
    got = raw.view(torch.bfloat16).to(torch.float64).numpy().reshape(T, D)
    ref = O.layer_norm(x_bf, c.layers[0]["ln1_g"], c.layers[0]["ln1_b"])
    err = np.abs(got - ref)
    bound = 2.0 ** -7 * np.abs(ref) + 1e-6
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{len(bad)} elements off, first at row {bad[0][0]}: {got[tuple(bad[0])]} vs {ref[tuple(bad[0])]}"
