"""Pins of the dense-layer oracle (oracle/linear.py) on CPU.

Each check is a consequence of y = x W^T + b that does not retype it: a
hand-worked example, the identity layer, a pure-Python triple loop, linearity,
and the packed (B, T, 3, H, D) order of the c_attn output read through a
selection layer. Broken copies of the oracle defined here (transposed weight,
bias dropped, heads and slots swapped) must each fail one of them.
"""

import json
import os

import numpy as np
import pytest

from oracle import linear as lin

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "linear_2x3_closed_form.json")


def _brute(x, w, b):
    M, K = len(x), len(x[0])
    N = len(w)
    y = [[0.0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(x[m][k]) * float(w[n][k])
            y[m][n] = acc + float(b[n])
    return np.array(y)


def pin_hand_worked(linear):
    g = json.load(open(GOLDEN))
    y = linear(np.array(g["x"]), np.array(g["w"]), np.array(g["b"]))
    assert np.array_equal(y, np.array(g["y"], dtype=np.float64)), "hand-worked 2x3"


def pin_identity(linear):
    r = np.random.default_rng(4)
    x = r.standard_normal((5, 6))
    b = r.standard_normal(6)
    assert np.array_equal(linear(x, np.eye(6), np.zeros(6)), x), "identity layer"
    assert np.array_equal(linear(x, np.eye(6), b), x + b), "identity layer + bias"


def pin_brute_force(linear):
    r = np.random.default_rng(5)
    for M, K, N in ((1, 1, 1), (3, 5, 4), (7, 2, 9)):
        x, w, b = r.standard_normal((M, K)), r.standard_normal((N, K)), r.standard_normal(N)
        assert np.allclose(linear(x, w, b), _brute(x.tolist(), w.tolist(), b.tolist()),
                           rtol=0, atol=1e-12), "triple loop"


def pin_linearity(linear):
    r = np.random.default_rng(6)
    x, x2 = r.standard_normal((4, 8)), r.standard_normal((4, 8))
    w, w2 = r.standard_normal((3, 8)), r.standard_normal((3, 8))
    b, z = r.standard_normal(3), np.zeros(3)
    assert np.allclose(linear(x + x2, w, z), linear(x, w, z) + linear(x2, w, z), atol=1e-12)
    assert np.allclose(linear(x, w + w2, z), linear(x, w, z) + linear(x, w2, z), atol=1e-12)
    assert np.allclose(linear(x, w, b) - linear(x, w, z), np.broadcast_to(b, (4, 3)), atol=1e-12)


def pin_packed_qkv_order(qkv_projection):
    """A selection layer: row r of W picks input column r mod C, and the bias
    is r itself, so qkv[b, t, s, h, d] = x[b, t, h*D + d] + (s*C + h*D + d)."""
    B, T, H, D = 2, 3, 4, 5
    C = H * D
    r = np.random.default_rng(7)
    x = r.standard_normal((B, T, C))
    w = np.zeros((3 * C, C))
    w[np.arange(3 * C), np.arange(3 * C) % C] = 1.0
    bias = np.arange(3 * C, dtype=np.float64)
    qkv = qkv_projection(x, w, bias, H)
    assert qkv.shape == (B, T, 3, H, D)
    s, h, d = np.meshgrid(np.arange(3), np.arange(H), np.arange(D), indexing="ij")
    expect = x[:, :, h * D + d] + (s * C + h * D + d)
    assert np.array_equal(qkv, expect), "packed (B, T, 3, H, D) order"


def test_oracle_meets_every_pin():
    pin_hand_worked(lin.linear)
    pin_identity(lin.linear)
    pin_brute_force(lin.linear)
    pin_linearity(lin.linear)
    pin_packed_qkv_order(lin.qkv_projection)


def test_output_projection_is_linear_on_the_flattened_heads():
    r = np.random.default_rng(8)
    out = r.standard_normal((2, 3, 4, 5))
    w, b = r.standard_normal((20, 20)), r.standard_normal(20)
    y = lin.output_projection(out, w, b)
    assert np.allclose(y.reshape(6, 20), _brute(out.reshape(6, 20).tolist(), w.tolist(),
                                                b.tolist()), atol=1e-12)


def _transposed(x, w, b):
    return np.asarray(x, np.float64) @ np.asarray(w, np.float64) + b


def _no_bias(x, w, b):
    return np.asarray(x, np.float64) @ np.asarray(w, np.float64).T


def _heads_before_slots(x, w, b, H):
    y = lin.linear(np.asarray(x).reshape(-1, x.shape[-1]), w, b)
    B, T, C = x.shape
    return y.reshape(B, T, H, 3, C // H).transpose(0, 1, 3, 2, 4)


@pytest.mark.parametrize("broken,pin", [
    (_transposed, "linear"),
    (_no_bias, "linear"),
    (_heads_before_slots, "qkv"),
])
def test_planted_mistakes_fail_a_pin(broken, pin):
    failed = False
    pins = ([pin_hand_worked, pin_identity, pin_brute_force, pin_linearity] if pin == "linear"
            else [pin_packed_qkv_order])
    for p in pins:
        try:
            p(broken)
        except (AssertionError, ValueError):
            failed = True
    assert failed
