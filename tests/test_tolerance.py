"""The out tolerance helper of the GPU parity tests (CPU only)."""

import numpy as np

from .test_parity_gpu import bf16_brackets, bf16_floor, out_error_ok, out_error_ok_faithful


def test_floor_is_the_bf16_half_spacing():
    o = np.array([0.3, 1.99, 3.9, 4.019755564672164])
    f = bf16_floor(o)
    assert np.all(f[:2] <= 2.0 ** -8)   # spacing 2^-7 in [1, 2)
    assert f[2] <= 2.0 ** -7            # spacing 2^-6 in [2, 4)
    # In [4, 8) the spacing is 2^-5: 4.0197... lies 0.0115 from 4.03125.
    assert abs(f[3] - (4.03125 - 4.019755564672164)) < 1e-15
    assert f[3] > 1e-2


def test_bound_is_1e2_where_representable():
    o = np.array([0.5, -1.25, 2.0])
    assert out_error_ok(o + 0.0099, o)[0]
    assert not out_error_ok(o + 0.0101, o)[0]


def test_floor_element_accepts_only_the_rounding_floor():
    o = np.array([4.019755564672164])   # nearest bf16 is 4.03125, 0.0115 away
    assert out_error_ok(np.array([4.03125]), o)[0]
    assert not out_error_ok(np.array([4.0]), o)[0]
    assert not out_error_ok(np.array([4.0625]), o)[0]


def test_brackets_enclose_the_value():
    lo, hi = bf16_brackets(np.array([4.019755564672164, 1.0, -4.019755564672164]))
    assert lo[0] == 4.0 and hi[0] == 4.03125
    assert lo[1] == hi[1] == 1.0
    assert lo[2] == -4.03125 and hi[2] == -4.0


def test_faithful_rule_admits_only_the_two_enclosing_values_at_the_floor():
    o = np.array([4.019755564672164])   # enclosed by 4.0 and 4.03125
    assert out_error_ok_faithful(np.array([4.03125]), o)[0]
    assert out_error_ok_faithful(np.array([4.0]), o)[0]
    assert not out_error_ok_faithful(np.array([4.0625]), o)[0]
    assert not out_error_ok_faithful(np.array([3.96875]), o)[0]
    # Where a bf16 lies within 1e-2 the bound stays 1e-2.
    r = np.array([0.5, -1.25, 2.0])
    assert out_error_ok_faithful(r + 0.0099, r)[0]
    assert not out_error_ok_faithful(r + 0.0101, r)[0]
