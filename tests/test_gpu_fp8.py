"""FP8 (e4m3) linear layers on the GPU through the C ABI against the oracle:
the per-row codes and scales bit for bit (decided in float32 on both sides),
and the tcgen05 kind::f8f6f4 GEMM against the oracle's sum of the same code
products (float64) scaled per row and column, at the QKV shape (512 -> 1536)
and both expert shapes (512 -> 1024, 1024 -> 512), with ragged row counts
that end inside a 256-row tile."""
import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O
from packed_sequence_transformer_b200 import ptl
from tests.gpu_util import dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    ptl.lib()


def _codes_host(t):
    """e4m3 codes (uint8 device tensor) as float64 values."""
    return t.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
@pytest.mark.parametrize("rows,cols", [(1, 512), (300, 512), (6823, 1024)])
def test_quantize_rows_bit_exact(dt, rows, cols):
    rng = np.random.default_rng(rows + cols)
    x = (rng.standard_normal((rows, cols)) * 2.0 ** rng.integers(-6, 6, (rows, 1))).astype(np.float32)
    x[0, :] = 0.0 if rows > 1 else x[0, :]
    td = torch.bfloat16 if dt == "bf16" else torch.float32
    xd = dev(x, td)
    xh = host(xd)  # the values the kernel sees (bf16-rounded in the bf16 build)
    codes, scales = ptl.quantize_rows_e4m3(xd)
    torch.cuda.synchronize()
    want_c, want_s = O.quantize_rows_e4m3(xh, precision="f32")
    np.testing.assert_array_equal(scales.cpu().numpy().astype(np.float64), want_s)
    np.testing.assert_array_equal(_codes_host(codes), want_c)


@pytest.mark.parametrize("M,K,N", [(6823, 512, 1536), (300, 512, 1024), (257, 1024, 512), (1, 128, 256),
                                   (300, 14336, 512)])
def test_linear_fp8_against_the_oracle(M, K, N):
    rng = np.random.default_rng(M + K + N)
    x = rng.standard_normal((M, K)).astype(np.float32)
    w = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    b = (0.02 * rng.standard_normal(N)).astype(np.float32)
    xd, wd = dev(x, torch.bfloat16), dev(w, torch.bfloat16)
    xq, sx = ptl.quantize_rows_e4m3(xd)
    wq, sw = ptl.quantize_rows_e4m3(wd)
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ptl.linear_fp8(xq, sx, wq, sw, dev(b, torch.float32), out, ws)
    torch.cuda.synchronize()
    assert ptl.last_device_error(ws) == 0
    g = host(out)
    # the oracle on the same (bf16) operands, codes decided in float32
    ref = O.linear_fp8(host(xd), host(wd), b, precision="f32")
    # float32 accumulation of K exact code products, then one bf16 rounding
    qx, qsx = O.quantize_rows_e4m3(host(xd), precision="f32")
    qw, qsw = O.quantize_rows_e4m3(host(wd), precision="f32")
    mag = (np.abs(qx) @ np.abs(qw).T) * qsx[:, None] * qsw[None, :]
    bound = K * 2.0 ** -24 * mag + 2.0 ** -8 * np.abs(ref) + 1e-30
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g))
    assert np.all(err <= bound), float((err / bound).max())
    # and the FP8 layer is an approximation of the bf16 one within e4m3 error
    exact = O.linear(host(xd), host(wd), b)
    assert np.max(np.abs(g - exact)) < 0.1 * np.max(np.abs(exact - b))


def test_linear_fp8_rejects_bad_shapes():
    L = ptl.lib()
    code = ptl.STATUS_CODE["PTL_ERR_SHAPE"]
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    p = ws.data_ptr()
    assert L.ptl_linear_fp8(p, p, p, p, None, p, 10, 100, 256, p, 256, None) == code   # K % 128
    assert L.ptl_linear_fp8(p, p, p, p, None, p, 10, 128, 200, p, 256, None) == code   # N % 256
    assert L.ptl_quantize_rows_e4m3(p, 1, 10, 24, p, p, None) == code                    # cols % 16
