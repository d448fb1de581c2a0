"""Pins for the oracle's FP8 (e4m3) operand quantisation and dequantised
GEMM, the reference for FP8 expert and QKV GEMMs: torch's float8_e4m3fn
conversion as the library routine for the rounding, the format's closed
forms (127 non-negative values, 448 the largest, spacing 2^-9 below 2^-6),
error bounds, and saturation (the reading taken for values beyond 448, where
the format itself has no infinity).  CPU only."""
import numpy as np
import pytest
import torch

from oracle import ptl_oracle as O


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float64)).to(torch.float8_e4m3fn).double().numpy()


def test_rounding_matches_torch_float8_e4m3fn():
    rng = np.random.default_rng(1)
    # many binades, both signs, subnormals, and exact ties between neighbours
    x = np.concatenate([
        rng.standard_normal(20000) * 2.0 ** rng.integers(-12, 9, 20000),
        np.array([1 + 1 / 16, 1 + 3 / 16, 2 ** -7 + 2 ** -10, 3 * 2 ** -10, 0.0, -0.0]),
    ])
    x = np.clip(x, -448, 448)
    np.testing.assert_array_equal(O.quantize_e4m3(x), _torch_e4m3(x))


def test_value_set_and_extremes():
    grid = np.unique(O.quantize_e4m3(np.linspace(0, 448, 400001)))
    assert grid.size == 127  # 16 exponents x 8 mantissas, less the NaN code
    assert grid.max() == 448.0 and grid[1] == 2.0 ** -9  # smallest subnormal
    sub = grid[(grid > 0) & (grid < 2.0 ** -6)]
    np.testing.assert_array_equal(sub, np.arange(1, 8) * 2.0 ** -9)
    # saturation beyond the largest finite value
    np.testing.assert_array_equal(O.quantize_e4m3([449.0, 1e6, -1e30]), [448.0, 448.0, -448.0])


def test_error_bounds_and_idempotence():
    rng = np.random.default_rng(2)
    x = rng.uniform(-448, 448, 50000) * 2.0 ** rng.integers(-16, 1, 50000)
    q = O.quantize_e4m3(x)
    normal = np.abs(x) >= 2.0 ** -6
    assert np.all(np.abs(q - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal])   # half of the 2^-3 spacing
    assert np.all(np.abs(q - x)[~normal] <= 2.0 ** -10)
    np.testing.assert_array_equal(O.quantize_e4m3(q), q)


def test_row_scaling():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((16, 300))
    x[3] = 0.0
    codes, s = O.quantize_rows_e4m3(x)
    assert s[3] == 1.0 and not codes[3].any()
    rows = np.arange(16) != 3
    # each row's largest magnitude maps to the largest code exactly
    np.testing.assert_array_equal(np.abs(codes[rows]).max(axis=1), np.full(15, 448.0))
    assert np.all(np.abs(codes * s[:, None] - x) <= 2.0 ** -4 * np.abs(x) + 2.0 ** -10 * s[:, None])


@pytest.mark.parametrize("K", [64, 512, 1024])
def test_fp8_linear_within_its_error_bound(K):
    rng = np.random.default_rng(K)
    x = rng.standard_normal((40, K))
    w = 0.02 * rng.standard_normal((24, K))
    b = rng.standard_normal(24)
    y8 = O.linear_fp8(x, w, b)
    y = O.linear(x, w, b)
    # each product carries at most (1 + 2^-4)^2 - 1 relative error from the
    # two roundings, plus the subnormal floor of each operand
    qx, sx = O.quantize_rows_e4m3(x)
    qw, sw = O.quantize_rows_e4m3(w)
    rel = (1 + 2.0 ** -4) ** 2 - 1
    floor = (2.0 ** -10 * sx[:, None]) * np.abs(w).sum(1)[None, :] + (2.0 ** -10 * sw[None, :]) * np.abs(x).sum(1)[:, None] \
        + 2.0 ** -20 * sx[:, None] * sw[None, :] * K
    bound = rel * (np.abs(x) @ np.abs(w).T) + floor
    assert np.all(np.abs(y8 - y) <= bound)
    # and it is a real approximation: far closer than the operands' size
    assert np.max(np.abs(y8 - y)) < 0.1 * np.max(np.abs(y - b))


def test_float32_decided_codes():
    """precision='f32': the scale is the float32 quotient max|row| / 448 and
    each code is the e4m3 rounding of the float32 quotient x / s; it differs
    from the float64-decided code only where the float64 quotient lies within
    one float32 rounding of a point halfway between two e4m3 neighbours, and
    then by exactly one e4m3 step."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 512)) * 2.0 ** rng.integers(-8, 8, (64, 1))).astype(np.float32)
    x[7] = 0.0
    c32, s32 = O.quantize_rows_e4m3(x, precision="f32")
    c64, s64 = O.quantize_rows_e4m3(x.astype(np.float64))
    amax = np.abs(x).max(axis=1).astype(np.float32)
    want_s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0))
    np.testing.assert_array_equal(s32, want_s.astype(np.float64))
    assert s32[7] == 1.0 and not c32[7].any()
    np.testing.assert_allclose(s32, s64, rtol=2.0 ** -23, atol=0)
    q32 = (x / want_s[:, None].astype(np.float32)).astype(np.float64)
    np.testing.assert_array_equal(c32, O.quantize_e4m3(q32))
    diff = c32 != c64
    assert diff.mean() < 1e-3
    # where they differ, the float64 quotient sits next to a rounding boundary
    q64 = x.astype(np.float64) / s64[:, None]
    a = np.abs(q64[diff])
    step = np.where(a >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -6))) - 3), 2.0 ** -9)
    frac = a / step - np.floor(a / step)
    assert np.all(np.abs(frac - 0.5) <= 2.0 ** -20 * a / step + 1e-9)
    assert np.all(np.abs(np.abs(c32[diff]) - np.abs(c64[diff])) <= step * (1 + 1e-12))
