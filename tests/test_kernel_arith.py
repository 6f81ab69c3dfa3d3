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


def _bf16_rne(x):
    """float32 -> bf16 (as float32) with round to nearest even."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def pack_f16_nonneg_model(p):
    """float32/uint32 restatement of pack_f16_nonneg for one value: times
    kF32ToF16Scale in fp32, keep bits [13, 29) of the product."""
    s = _const("kF32ToF16Scale")
    m = (np.asarray(p, dtype=np.float32) * s).astype(np.float32)
    b = m.view(np.uint32).astype(np.uint64) >> 13
    assert np.all(b < 0x8000)   # no carry into the other half of the pair
    return b.astype(np.uint16).view(np.float16)


def test_f16_pack_scale():
    # 2^-112 moves the exponent bias from 127 to 15; (1 + 3 * 2^-13) is the
    # rounding bias, exact in fp32.
    assert float(_const("kF32ToF16Scale")) == 2.0 ** -112 * (1 + 3 * 2.0 ** -13)


def _fp16_neighbours(x):
    """The fp16 values just below-or-at and just above x (x >= 2^-14, normal)."""
    x = np.asarray(x, np.float64)
    ulp = 2.0 ** (np.floor(np.log2(x)) - 10)
    lo = np.floor(x / ulp) * ulp
    return lo, lo + ulp, ulp


def test_f16_pack_rounds_faithfully_with_the_stated_threshold():
    # Probabilities in [2^-14, 2^8] (fp16 normals; 2^8 is the stale-max bound).
    rng = np.random.default_rng(0)
    p = np.exp2(rng.uniform(-14, 8, 400_000)).astype(np.float32)
    got = pack_f16_nonneg_model(p).astype(np.float64)
    x = p.astype(np.float64)
    lo, hi, ulp = _fp16_neighbours(x)
    # One of the two fp16 values around p, error below 3/4 of a unit.
    assert np.all((got == lo) | (got == hi))
    assert np.all(np.abs(got - x) <= 0.75 * ulp)
    # Up exactly when the dropped part exceeds 1 - 3f/8 units, f the
    # significand (checked away from the threshold, where the fp32 product's
    # own rounding cannot decide).
    f = x / (2.0 ** np.floor(np.log2(x)))
    frac = (x - lo) / ulp
    thr = 1.0 - 3.0 * f / 8.0
    clear = np.abs(frac - thr) > 2.0 ** -8
    assert np.all(got[clear] == np.where(frac[clear] > thr[clear], hi[clear], lo[clear]))
    # fp16 values stay themselves.
    exact = np.exp2(rng.uniform(-14, 8, 10_000)).astype(np.float16).astype(np.float32)
    assert np.array_equal(pack_f16_nonneg_model(exact).astype(np.float32), exact)
    # The mean error over p log-uniform across the range: 3/8 E[f] - 1/2 =
    # 3 / (8 ln 2) - 1/2 = +0.041 of a unit (plain truncation gives -1/2).
    assert abs(np.mean((got - x) / ulp) - (3 / (8 * np.log(2)) - 0.5)) < 0.005


def test_f16_pack_below_the_normal_range():
    # Below 2^-14 the fp32 product is denormal: the result stays within one
    # fp16 subnormal unit (2^-24) of p, and 0 maps to 0.
    rng = np.random.default_rng(1)
    p = np.concatenate([rng.uniform(0, 2.0 ** -14, 50_000), [0.0, 2.0 ** -24]]).astype(np.float32)
    got = pack_f16_nonneg_model(p).astype(np.float64)
    assert np.all(np.abs(got - p.astype(np.float64)) < 2.0 ** -24)
    assert float(pack_f16_nonneg_model(np.float32(0.0))) == 0.0


def split3_bf16_model(v):
    """float32 restatement of split3_bf16: three bf16 terms whose sum is v."""
    v = np.asarray(v, dtype=np.float32)
    h1 = _bf16_rne(v)
    r1 = (v - h1).astype(np.float32)
    h2 = _bf16_rne(r1)
    h3 = _bf16_rne((r1 - h2).astype(np.float32))
    return h1, h2, h3


def test_split3_bf16_recovers_fp32_constants():
    # The per-query constants folded into the dK/dV products (-lse*log2e-like
    # values up to ~1e3 and -Delta): the three bf16 terms sum to v within
    # 2^-24 of |v| in exact arithmetic, as the tensor core accumulates them.
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(0, 30, 100_000), rng.uniform(-1500, 1500, 100_000),
                        rng.normal(0, 1e-3, 10_000)]).astype(np.float32)
    h1, h2, h3 = split3_bf16_model(v)
    total = h1.astype(np.float64) + h2.astype(np.float64) + h3.astype(np.float64)
    err = np.abs(total - v.astype(np.float64))
    assert np.all(err <= 2.0 ** -24 * np.abs(v.astype(np.float64)))


def bf16x2_to_f16x2_model(u):
    """uint32 restatement of bf16x2_to_f16x2 on packed pairs: magnitude mask,
    per-half unsigned max with 0x3800 (clamp), one 32-bit multiply-add
    (mag * 8 + 0x3FFE4000 mod 2^32), signs put back. Returns the packed fp16
    pairs and the per-half magnitudes the range tracker sees."""
    u = np.asarray(u, dtype=np.uint32)
    mag = u & np.uint32(0x7FFF7FFF)
    lo = np.maximum(mag & np.uint32(0xFFFF), np.uint32(0x3800))
    hi = np.maximum(mag >> np.uint32(16), np.uint32(0x3800))
    clamped = (hi << np.uint32(16)) | lo
    z = (clamped.astype(np.uint64) * 8 + 0x3FFE4000) & 0xFFFFFFFF
    r = z.astype(np.uint32) | (u & np.uint32(0x80008000))
    return r, mag & np.uint32(0xFFFF), mag >> np.uint32(16)


def _check_halves(v, h):
    """Every in-range bf16 value v against the fp16 value h it became."""
    v = v.astype(np.float64)
    h = h.astype(np.float64)
    normal = np.abs(v) >= 2.0 ** -14
    assert np.all(h[normal] == v[normal])                     # exact
    tiny = ~normal
    assert np.all(np.abs(h[tiny] - v[tiny]) <= 2.0 ** -15)    # within 2^-15
    assert np.all(h[np.abs(v) < 2.0 ** -15] == 0)             # flushed to +-0
    assert np.all(np.signbit(h) == np.signbit(v))


def test_v_conversion_bf16_to_fp16_over_every_bf16_value():
    # The forward rewrites V from bf16 to fp16 with integer operations only.
    # Over all 65536 bf16 patterns, in the low and in the high half of a word
    # (with an in-range partner in the other half): every |v| <= 65280 (the
    # largest bf16 fp16 holds) converts exactly down to 2^-14 and within 2^-15
    # below; the partner is unaffected; and exactly the patterns beyond that
    # (|v| >= 65536, inf, NaN) raise the range tracker.
    bits = np.arange(65536, dtype=np.uint32)
    v = (bits << np.uint32(16)).view(np.float32)
    in_range = np.isfinite(v) & (np.abs(v) <= 65280.0)
    partner = np.uint32(0xBF40)                             # -0.75
    for shift in (0, 16):
        other = 16 - shift
        words = (bits << np.uint32(shift)) | (partner << np.uint32(other))
        r, mlo, mhi = bf16x2_to_f16x2_model(words)
        m = mlo if shift == 0 else mhi
        flagged = m >= 0x4780                                 # kBf16BeyondF16
        assert np.array_equal(flagged, ~in_range)
        h = ((r >> np.uint32(shift)) & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16)
        _check_halves(v[in_range], h[in_range])
        p = ((r[in_range] >> np.uint32(other)) & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16)
        assert np.all(p.astype(np.float64) == -0.75)
    # Boundary values: 65280 converts exactly, 65536 is flagged.
    r, mlo, _ = bf16x2_to_f16x2_model(np.array([0x477F, 0x4780], dtype=np.uint32))
    assert (r[0] & 0xFFFF).astype(np.uint16).view(np.float16) == 65280.0
    assert mlo[0] < 0x4780 <= mlo[1]


def test_v_conversion_random_pairs_both_halves():
    # Random in-range pairs: both halves exact (or within 2^-15 when tiny).
    rng = np.random.default_rng(3)
    f = np.concatenate([rng.normal(0, 1, 200_000), rng.normal(0, 1e-4, 20_000),
                        rng.uniform(-65280, 65280, 20_000)]).astype(np.float32)
    b = (f.view(np.uint32) >> np.uint32(16)).astype(np.uint32)     # truncate to bf16
    b = b[: (len(b) // 2) * 2].reshape(-1, 2)
    words = b[:, 0] | (b[:, 1] << np.uint32(16))
    r, mlo, mhi = bf16x2_to_f16x2_model(words)
    assert np.all(mlo < 0x4780) and np.all(mhi < 0x4780)
    for k, shift in enumerate((0, 16)):
        v = (b[:, k] << np.uint32(16)).view(np.float32)
        h = ((r >> np.uint32(shift)) & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16)
        _check_halves(v, h)
