"""Checks that pin a causal-attention implementation to what the definition fixes.

Each pin takes the implementation under test as two callables:

    fwd(qkv, scale)        -> (out (B,T,H,D), lse (B,H,T))
    fwdbwd(qkv, dout, scale) -> (out, lse, dqkv (B,T,3,H,D))

and raises AssertionError when the implementation breaks the property.
The same pins run against the fp64 oracle (where they must all pass) and
against deliberately broken copies of it defined in the tests (where at least
one must fail). None of them retypes the oracle's formula: each checks a
consequence of the definition (a closed form, an invariant, a limit or a
finite difference).
"""

from __future__ import annotations

import numpy as np


def _rng(seed):
    return np.random.default_rng(seed)


def pin_row_sums_and_support(probabilities):
    """Every probability row sums to 1 and puts no weight on future keys.

    ``probabilities(Q, K, scale) -> P (T, T)``.
    """
    r = _rng(1)
    for T, D in ((1, 4), (7, 4), (33, 16)):
        Q = r.standard_normal((T, D))
        K = r.standard_normal((T, D))
        P = probabilities(Q, K, 0.25)
        assert np.all(np.abs(P.sum(axis=1) - 1.0) <= 1e-12), "row sums"
        assert np.all(P[np.triu_indices(T, k=1)] == 0.0), "weight on future keys"
        assert np.all(P >= 0.0)


def pin_query_zero(fwd):
    """Query 0 sees only key 0: out[t=0] == v[t=0] exactly, lse = s_00."""
    r = _rng(2)
    B, T, H, D = 2, 9, 3, 8
    qkv = r.standard_normal((B, T, 3, H, D))
    scale = 0.3
    out, lse = fwd(qkv, scale)
    assert np.array_equal(out[:, 0], qkv[:, 0, 2]), "out[0] != V[0]"
    s00 = scale * np.einsum("bhd,bhd->bh", qkv[:, 0, 0], qkv[:, 0, 1])
    assert np.allclose(lse[:, :, 0], s00, rtol=0, atol=1e-14), "lse[0] != s_00"


def pin_zero_queries_prefix_mean(fwd):
    """With Q = 0 every visible logit is 0: out_i = mean(v_0..v_i), lse_i = ln(i+1)."""
    r = _rng(3)
    B, T, H, D = 1, 17, 2, 5
    qkv = r.standard_normal((B, T, 3, H, D))
    qkv[:, :, 0] = 0.0
    out, lse = fwd(qkv, 0.125)
    v = qkv[:, :, 2]
    prefix = np.cumsum(v, axis=1) / np.arange(1, T + 1)[None, :, None, None]
    assert np.allclose(out, prefix, rtol=0, atol=1e-12), "prefix mean"
    want = np.log(np.arange(1, T + 1, dtype=np.float64))
    assert np.allclose(lse, np.broadcast_to(want, lse.shape), rtol=0, atol=1e-12), "lse = ln(i+1)"


def pin_single_token(fwdbwd):
    """T = 1: out = v, lse = scale q.k, dV = dO and dQ = dK = 0 (P is 1)."""
    r = _rng(4)
    B, T, H, D = 3, 1, 2, 6
    qkv = r.standard_normal((B, T, 3, H, D))
    dout = r.standard_normal((B, T, H, D))
    scale = 0.7
    out, lse, dqkv = fwdbwd(qkv, dout, scale)
    assert np.allclose(out, qkv[:, :, 2], rtol=0, atol=1e-14)
    s = scale * np.einsum("bthd,bthd->bht", qkv[:, :, 0], qkv[:, :, 1])
    assert np.allclose(lse, s, rtol=0, atol=1e-14)
    assert np.allclose(dqkv[:, :, 2], dout, rtol=0, atol=1e-14), "dV != dO"
    assert np.allclose(dqkv[:, :, 0:2], 0.0, rtol=0, atol=1e-14), "dQ, dK != 0"


def pin_key_shift(fwdbwd):
    """Adding one vector u to every key leaves out and dV unchanged and shifts
    lse_i by scale * q_i . u. The key gradients then sum to zero over keys,
    because each logit row moves by a constant."""
    r = _rng(5)
    B, T, H, D = 1, 12, 2, 4
    qkv = r.standard_normal((B, T, 3, H, D))
    dout = r.standard_normal((B, T, H, D))
    scale = 0.5
    u = r.standard_normal((H, D))
    shifted = qkv.copy()
    shifted[:, :, 1] += u[None, None]
    o1, l1, g1 = fwdbwd(qkv, dout, scale)
    o2, l2, g2 = fwdbwd(shifted, dout, scale)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12), "out moved under key shift"
    dl = scale * np.einsum("bthd,hd->bht", qkv[:, :, 0], u)
    assert np.allclose(l2 - l1, dl, rtol=0, atol=1e-12), "lse shift"
    assert np.allclose(g1[:, :, 2], g2[:, :, 2], rtol=0, atol=1e-12), "dV moved"
    assert np.allclose(g1[:, :, 1].sum(axis=1), 0.0, rtol=0, atol=1e-12), "sum_j dK_j != 0"


def pin_finite_differences(fwdbwd):
    """Central differences of L = sum(dO * out) on H=1, T=8, D=4, scale=0.5.

    Every one of the 96 qkv entries must match the analytic gradient to
    1e-6 * max(1, |g|) with step h = 1e-6 in fp64.
    """
    r = _rng(6)
    B, T, H, D = 1, 8, 1, 4
    qkv = r.standard_normal((B, T, 3, H, D))
    dout = r.standard_normal((B, T, H, D))
    scale = 0.5
    _, _, g = fwdbwd(qkv, dout, scale)

    def loss(x):
        o, _, _ = fwdbwd(x, dout, scale)
        return float(np.sum(o * dout))

    h = 1e-6
    for idx in np.ndindex(qkv.shape):
        xp = qkv.copy()
        xm = qkv.copy()
        xp[idx] += h
        xm[idx] -= h
        fd = (loss(xp) - loss(xm)) / (2 * h)
        assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(g[idx])), (idx, fd, g[idx])


def pin_closed_form_fixture(fwdbwd, fixture):
    """Hand-worked T=3 example with exact answers (tests/golden)."""
    ev = _fixture_eval
    q = ev(fixture["q"])
    k = ev(fixture["k"])
    v = ev(fixture["v"])
    do = ev(fixture["do"])
    scale = float(ev(fixture["scale"]))
    T, D = q.shape
    qkv = np.stack([q, k, v], axis=1)[None, :, :, None, :]  # (1,T,3,1,D)
    dout = do[None, :, None, :]
    out, lse, dqkv = fwdbwd(qkv, dout, scale)
    e = fixture["expected"]
    tol = dict(rtol=0, atol=1e-14)
    assert np.allclose(out[0, :, 0], ev(e["o"]), **tol), "o"
    assert np.allclose(lse[0, 0], ev(e["lse"]), **tol), "lse"
    assert np.allclose(dqkv[0, :, 2, 0], ev(e["dv"]), **tol), "dv"
    assert np.allclose(dqkv[0, :, 0, 0], ev(e["dq"]), **tol), "dq"
    assert np.allclose(dqkv[0, :, 1, 0], ev(e["dk"]), **tol), "dk"


def _fixture_eval(x):
    import math

    env = {"ln": math.log, "__builtins__": {}}
    if isinstance(x, str):
        return float(eval(x, env))  # committed fixture, arithmetic only
    return np.array([_fixture_eval(y) for y in x], dtype=np.float64)
