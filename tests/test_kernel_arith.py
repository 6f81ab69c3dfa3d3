"""CPU checks of bit-level arithmetic the kernels use instead of library calls.

Each test restates one device helper step by step in numpy float32/uint32 and
checks it against the exact mathematics. The coefficients are read from the
kernel source, so a changed constant is tested as compiled.
"""

import os
import re

import numpy as np

PTX = os.path.join(os.path.dirname(__file__), "..", "causal_self_attention_flashattention_b200",
                   "csrc", "ptx.cuh")


def _const(name):
    src = open(PTX).read()
    m = re.search(r"constexpr float %s = ([0-9.eE+-]+)f;" % name, src)
    assert m, name
    return np.float32(float(m.group(1)))


def exp2_poly_model(y):
    """float32 restatement of exp2_poly2 (one lane): clamp, rint by adding
    1.5*2^23, cubic in f = y - n by Horner's rule, then n added to the exponent
    bits (as bits(t) << 23)."""
    y = np.asarray(y, dtype=np.float32)
    c0, c1, c2, c3 = (_const("kExp2Poly%d" % i) for i in range(4))
    rnd = np.float32(12582912.0)
    a = np.maximum(y, np.float32(-125.0))
    t = (a + rnd).astype(np.float32)
    n = (t - rnd).astype(np.float32)
    f = (a - n).astype(np.float32)                       # fma(n, -1, a) is exact here
    q = (f * c3 + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error():
    # Every exponent the softmax can produce: y <= 8 (the stale-max bound).
    y = np.linspace(-124.0, 8.0, 400_001, dtype=np.float32)
    got = exp2_poly_model(y).astype(np.float64)
    ref = np.exp2(y.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_exp2_poly_integers_and_halves():
    # At integers f = 0 and the result is c0 * 2^n; at half-integers rint
    # rounds to even, so f = +-1/2 both occur.
    y = np.array([-3.0, 0.0, 1.0, 7.0, -2.5, -1.5, 0.5], dtype=np.float32)
    got = exp2_poly_model(y).astype(np.float64)
    assert np.allclose(got, np.exp2(y.astype(np.float64)), rtol=1e-4, atol=0)


def test_exp2_poly_masked_and_underflow_inputs():
    # -inf (masked scores) and very negative y are clamped: the result is a
    # tiny positive normal number, never negative, inf or NaN.
    y = np.array([-np.inf, -1e30, -300.0, -125.0, -124.9], dtype=np.float32)
    got = exp2_poly_model(y)
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got < 2.0 ** -123)
