"""Pins of the e4m3 quantiser the FP8 forward is checked with (oracle/fp8.py).

They check what the format and the per-tensor reading fix, not the code: the
e4m3 grid (every finite pattern round-trips, 448 is the largest, the spacing
near 1 is 2^-3), round-to-nearest-even at exact midpoints, that a tensor's
largest magnitude lands on +-448 exactly, the relative error bound of the
dequantised values, and the zero tensor.
"""

import numpy as np

from oracle import fp8


def _all_finite_patterns():
    b = np.arange(256, dtype=np.uint8)
    return b[(b & 0x7F) != 0x7F]          # 0x7F / 0xFF are NaN in e4m3fn


def test_grid_round_trips_and_bounds():
    b = _all_finite_patterns()
    v = fp8.e4m3_value(b)
    assert np.array_equal(fp8.e4m3_bits(v)[v != 0], b[v != 0])
    assert np.max(np.abs(v)) == 448.0
    pos = np.sort(v[v > 0])
    assert pos[0] == 2.0 ** -9                          # smallest subnormal
    one = np.searchsorted(pos, 1.0)
    assert pos[one] == 1.0 and pos[one + 1] == 1.125    # 3 mantissa bits


def test_midpoints_round_to_even():
    # 1.0625 lies halfway between 1.0 (mantissa 000) and 1.125 (001): even wins.
    assert fp8.e4m3_value(fp8.e4m3_bits(np.float32([1.0625])))[0] == 1.0
    # 1.1875 lies between 1.125 (001) and 1.25 (010): the even one is 1.25.
    assert fp8.e4m3_value(fp8.e4m3_bits(np.float32([1.1875])))[0] == 1.25
    assert fp8.e4m3_value(fp8.e4m3_bits(np.float32([-1.0625])))[0] == -1.0


def test_amax_lands_on_448_and_error_bound():
    r = np.random.default_rng(11)
    qkv = (r.standard_normal((2, 50, 3, 2, 64)) * np.array([1.0, 3.0, 0.5])[None, None, :, None, None]
           ).astype(np.float32)
    bits, dq = fp8.quantize_qkv(qkv)
    deq = fp8.dequantize_qkv(bits, dq)
    for s in range(3):
        x = qkv[:, :, s].astype(np.float64)
        k = np.unravel_index(np.argmax(np.abs(x)), x.shape)
        assert abs(fp8.e4m3_value(bits[:, :, s][k])) == 448.0
        # Normal e4m3 values (|x8| >= 2^-6) are within half a spacing, 2^-4
        # relative, of the scaled input; subnormals within 2^-10 absolute (in
        # scaled units); the fp32 scale steps add a few ulps.
        scaled = np.abs(x) * 448.0 / np.abs(x).max()
        err = np.abs(deq[:, :, s] - x) * 448.0 / np.abs(x).max()
        normal = scaled >= 2.0 ** -6
        assert np.all(err[normal] <= (2.0 ** -4 + 1e-6) * scaled[normal])
        assert np.all(err[~normal] <= 2.0 ** -10 + 1e-9)


def test_zero_tensor_quantises_to_zero_with_unit_scale():
    bits, dq = fp8.quantize_qkv(np.zeros((1, 4, 3, 1, 64), np.float32))
    assert np.all(bits == 0) and np.all(dq == 1.0)
