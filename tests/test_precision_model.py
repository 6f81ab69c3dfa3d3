"""Why the forward multiplies P and V in fp16: a float32 restatement of the
forward kernel's arithmetic, checked against the oracle on CPU.

The model follows the kernel step by step for one head: S = Q K^T in fp32
from bf16 inputs; per 128-key tile, the row max with the stale-max rule
(raised only when it grows by more than 2^8 in base 2), p = 2^(s*c - m*c)
with every 4th pair of columns on the FMA-pipe polynomial, the row sum in the
kernel's order, P packed to fp16 (round half up) and multiplied with V
converted to fp16, O rescaled when the max is raised; at the end
out = bf16(O / l) and lse = ln2 * (m*c + log2 l). Replacing the fp16 P and V
with bf16 shows what the precision choice buys.
"""

import numpy as np
import pytest

from oracle import oracle as orc
from causal_self_attention_flashattention_b200.workload import make_inputs

from .test_kernel_arith import _bf16_rne, exp2_poly_model, pack_f16_nonneg_model
from .test_parity_gpu import LSE_TOL, out_error_ok

LOG2E = 1.4426950408889634
POLY_COLS = np.array([(col // 2) % 4 == 3 for col in range(128)])


def kernel_forward_model(Q, K, V, scale, p_format="f16"):
    Q, K, V = (np.asarray(a, dtype=np.float32) for a in (Q, K, V))
    T, D = V.shape
    c = np.float32(np.float32(scale) * np.float32(LOG2E))
    S = (Q @ K.T).astype(np.float32)
    Vp = V.astype(np.float16).astype(np.float32) if p_format == "f16" else V
    m = np.full(T, -np.inf, np.float32)
    l = np.zeros(T, np.float32)
    O = np.zeros((T, D), np.float32)
    for j in range((T + 127) // 128):
        r0 = 128 * j
        rows = np.arange(r0, T)                       # query tiles i >= j
        cols = np.arange(r0, min(r0 + 128, T))
        x = np.full((len(rows), 128), -np.inf, np.float32)
        x[:, :len(cols)] = S[np.ix_(rows, cols)]
        x[(r0 + np.arange(128))[None, :] > rows[:, None]] = -np.inf   # future keys
        mx = x.max(axis=1)
        mr = m[rows]
        first = np.isneginf(mr)
        with np.errstate(invalid="ignore"):
            grow = first | ((mx - mr) * c > np.float32(8))
        m_new = np.where(grow, mx, mr).astype(np.float32)
        with np.errstate(invalid="ignore"):
            alpha = np.where(grow, np.exp2(((mr - m_new) * c).astype(np.float32)), 1)
        alpha = np.where(first, 0, alpha).astype(np.float32)
        neg_mc = (-m_new * c).astype(np.float32)
        # fma(s, c, -m*c) rounded once to fp32
        y = (x.astype(np.float64) * np.float64(c) + neg_mc[:, None]).astype(np.float32)
        p = np.exp2(y).astype(np.float32)              # ex2 of -inf is +0
        p[:, POLY_COLS] = exp2_poly_model(y[:, POLY_COLS])
        sa = np.zeros((len(rows), 4), np.float32)
        sb = np.zeros((len(rows), 4), np.float32)
        for c2 in range(64):
            sa[:, c2 & 3] += p[:, 2 * c2]
            sb[:, c2 & 3] += p[:, 2 * c2 + 1]
        s = ((sa[:, 0] + sb[:, 0]) + (sa[:, 1] + sb[:, 1])) + ((sa[:, 2] + sb[:, 2]) + (sa[:, 3] + sb[:, 3]))
        l[rows] = (l[rows] * alpha + s).astype(np.float32)
        pq = pack_f16_nonneg_model(p).astype(np.float32) if p_format == "f16" else _bf16_rne(p)
        vt = np.zeros((128, D), np.float32)
        vt[:len(cols)] = Vp[cols]
        O[rows] = (O[rows] * alpha[:, None] + pq @ vt).astype(np.float32)
        m[rows] = m_new
    out = _bf16_rne((O * (np.float32(1) / l)[:, None]).astype(np.float32))
    lse = (np.float32(np.log(2.0)) * (m * c + np.log2(l).astype(np.float32))).astype(np.float32)
    return out, lse


def _head(B, T, H, qk_std, b, h):
    qkv, _ = make_inputs(B, T, H, 64, seed=0, qk_std=qk_std)
    q64 = qkv.double().numpy()
    return tuple(q64[b, :, s, h] for s in range(3))


@pytest.mark.parametrize("B,T,H,qk_std,b,h", [
    (16, 1024, 12, 1.0, 0, 0),     # the bench workload
    (4, 4096, 12, 3.0, 3, 11),     # the stress workload's head with o = 4.0198
    (4, 4096, 12, 3.0, 0, 0),
])
def test_fp16_p_meets_the_tolerances(B, T, H, qk_std, b, h):
    Q, K, V = _head(B, T, H, qk_std, b, h)
    O, lse, _ = orc.head_forward(Q, K, V, 0.125)
    out, lse_m = kernel_forward_model(Q, K, V, 0.125, "f16")
    ok, err, _ = out_error_ok(out.astype(np.float64), O)
    assert ok, err
    assert np.max(np.abs(lse_m - lse)) <= LSE_TOL


def test_bf16_p_fails_the_stress_workload():
    # Peaked rows (q, k ~ N(0, 3^2)): one p near 1 times a large v. With P
    # and V in bf16 the out error passes 1e-2 where fp16 stays inside it.
    Q, K, V = _head(4, 4096, 12, 3.0, 0, 0)
    O, _, _ = orc.head_forward(Q, K, V, 0.125)
    ok16, err16, _ = out_error_ok(kernel_forward_model(Q, K, V, 0.125, "f16")[0].astype(np.float64), O)
    okb, errb, _ = out_error_ok(kernel_forward_model(Q, K, V, 0.125, "bf16")[0].astype(np.float64), O)
    assert ok16 and not okb
    assert errb > 1.2e-2 > err16
