"""Why the forward multiplies P and V in fp16: a float32 restatement of the
forward kernel's arithmetic, checked against the oracle on CPU.

The model follows the kernel step by step for one head: S = Q K^T in fp32
from bf16 inputs; per 128-key tile, the row max with the stale-max rule
(raised only when it grows by more than 2^8 in base 2), p = 2^(s*c - m*c)
with every 6th pair of columns on the FMA-pipe polynomial, the row sum in the
kernel's order, P packed to fp16 (the biased truncation of pack_f16_nonneg)
and multiplied with V converted to fp16 (the integer conversion: exact down
to 2^-14), O rescaled when the max is raised; at the end
out = bf16(O / l) and lse = ln2 * (m*c + log2 l). Replacing the fp16 P and V
with bf16 shows what the precision choice buys.
"""

import numpy as np
import pytest

from oracle import oracle as orc
from causal_self_attention_flashattention_b200.workload import make_inputs

from .test_kernel_arith import (_bf16_rne, bf16x2_to_f16x2_model, exp2_poly_model,
                                pack_f16_nonneg_model)
from .test_parity_gpu import LSE_TOL, out_error_ok

LOG2E = 1.4426950408889634
# The forward's kPolyEvery: pair c2 = col // 2 uses the polynomial when
# c2 % 6 == 5.
POLY_COLS = np.array([(col // 2) % 6 == 5 for col in range(128)])


def v_to_f16_model(V):
    """V (bf16 values held in float32) as the forward's integer conversion
    turns them into fp16, back in float32. Values that are not bf16 (the
    dequantized e4m3 inputs below) are rounded to fp16 directly."""
    bits = np.ascontiguousarray(V, dtype=np.float32).view(np.uint32)
    if np.any(bits & np.uint32(0xFFFF)):
        return np.asarray(V, np.float32).astype(np.float16).astype(np.float32)
    r, _, _ = bf16x2_to_f16x2_model((bits >> np.uint32(16)).ravel())
    h = (r & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16)
    return h.astype(np.float32).reshape(V.shape)


def kernel_forward_model(Q, K, V, scale, p_format="f16"):
    Q, K, V = (np.asarray(a, dtype=np.float32) for a in (Q, K, V))
    T, D = V.shape
    c = np.float32(np.float32(scale) * np.float32(LOG2E))
    S = (Q @ K.T).astype(np.float32)
    Vp = v_to_f16_model(V) if p_format == "f16" else V
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


def _fma32(a, b, c):
    """fp32 fused multiply-add: the exact a*b + c rounded once (two fp32
    factors multiply exactly in fp64; the sum is rounded in fp64 first, which
    differs from a single rounding only in rare ties)."""
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(np.float32)


def delta_model(dO, O):
    """Delta of every row as the dQ kernel sums it: each 16-column group in
    four fp32 accumulators (fused multiply-adds over the bf16 pairs), the
    group's sum as (a0 + a1) + (a2 + a3), then the four groups the same way."""
    dO = np.asarray(dO, np.float32)
    O = np.asarray(O, np.float32)
    parts = []
    for g in range(4):
        acc = [np.zeros(dO.shape[0], np.float32) for _ in range(4)]
        for e in range(8):                        # 8 words = 16 columns
            for half in (0, 1):
                col = 16 * g + 2 * e + half
                acc[e & 3] = _fma32(dO[:, col], O[:, col], acc[e & 3])
        parts.append((acc[0] + acc[1]) + (acc[2] + acc[3]))
    return (parts[0] + parts[1]) + (parts[2] + parts[3])


def kernel_backward_model(Q, K, V, dO, out, lse, scale, fold_terms=3):
    """fp32 restatement of the dQ and dK/dV kernels for one head (T a multiple
    of 128), from the forward's bf16 out and fp32 lse. dK/dV folds -lse/scale
    and -Delta into its products as `fold_terms` bf16 terms (3 in the kernel);
    P and dS go to the tensor core as bf16."""
    Q, K, V, dO, out = (np.asarray(a, np.float32) for a in (Q, K, V, dO, out))
    lse = np.asarray(lse, np.float32)
    T, D = Q.shape
    nt = T // 128
    sc = np.float32(np.float32(scale) * np.float32(LOG2E))
    delta = delta_model(dO, out)
    inv_scale = np.float32(1) / np.float32(scale)

    def fold(v):
        terms, r = [], v.astype(np.float32)
        for _ in range(fold_terms):
            t = _bf16_rne(r)
            terms.append(t)
            r = (r - t).astype(np.float32)
        return np.sum(np.stack(terms).astype(np.float64), axis=0)

    vl = fold((-lse * inv_scale).astype(np.float32))      # per query row
    vd = fold(-delta)
    nl = (-lse * np.float32(LOG2E)).astype(np.float32)
    nd = -delta
    dq = np.zeros((T, D), np.float32)
    dk = np.zeros((T, D), np.float32)
    dv = np.zeros((T, D), np.float32)
    for i in range(nt):                 # query tile
        qi, qs = slice(128 * i, 128 * i + 128), np.arange(128 * i, 128 * i + 128)
        for j in range(i + 1):          # key tile
            kj, ks = slice(128 * j, 128 * j + 128), np.arange(128 * j, 128 * j + 128)
            S = (Q[qi] @ K[kj].T).astype(np.float32)
            dP = (dO[qi] @ V[kj].T).astype(np.float32)
            future = ks[None, :] > qs[:, None]
            # dQ kernel: p = 2^(s*c - lse*log2e), dS = p * (dP - Delta)
            with np.errstate(over="ignore"):
                p_q = np.exp2(_fma32(S, sc, nl[qi, None]))
            p_q[future] = 0
            ds_q = _bf16_rne((p_q * (dP + nd[qi, None])).astype(np.float32))
            dq[qi] = (dq[qi] + ds_q @ K[kj]).astype(np.float32)
            # dK/dV kernel: the folded constants come out of the products
            s_f = (S.astype(np.float64) + vl[qi, None]).astype(np.float32)
            dp_f = (dP.astype(np.float64) + vd[qi, None]).astype(np.float32)
            with np.errstate(over="ignore"):
                p_k = np.exp2((s_f * sc).astype(np.float32))
            p_k[future] = 0
            pb = _bf16_rne(p_k)
            db = _bf16_rne((p_k * dp_f).astype(np.float32))
            dv[kj] = (dv[kj] + pb.T @ dO[qi]).astype(np.float32)
            dk[kj] = (dk[kj] + db.T @ Q[qi]).astype(np.float32)
    s = np.float32(scale)
    return _bf16_rne(dq * s), _bf16_rne(dk * s), _bf16_rne(dv)


def _rel_fro(g, o):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    return np.linalg.norm(g - o) / np.linalg.norm(o)


def _grads(B, T, H, qk_std, b, h, fold_terms=3):
    qkv, dout = make_inputs(B, T, H, 64, seed=0, qk_std=qk_std)
    q64, d64 = qkv.double().numpy(), dout.double().numpy()
    Q, K, V = (q64[b, :, s, h] for s in range(3))
    dO = d64[b, :, h]
    out, lse = kernel_forward_model(Q, K, V, 0.125, "f16")
    model = kernel_backward_model(Q, K, V, dO, out, lse, 0.125, fold_terms)
    ref = orc.head_backward(Q, K, V, dO, 0.125)
    return [_rel_fro(g, o) for g, o in zip(model, ref)]


@pytest.mark.parametrize("B,T,H,qk_std,b,h", [
    (16, 1024, 12, 1.0, 7, 5),      # the bench workload
    (4, 4096, 12, 3.0, 3, 11),      # the stress workload
])
def test_backward_arithmetic_meets_the_gradient_tolerance(B, T, H, qk_std, b, h):
    errs = _grads(B, T, H, qk_std, b, h)
    assert max(errs) <= 2e-2, errs


def test_one_term_fold_of_the_row_constants_would_not_do():
    # Folding -lse/scale as a single bf16 term (its rounding error is up to
    # 2^-9 of |lse|/scale, ~0.3 here) skews every P of the row; the three-term
    # split keeps it to 2^-24.
    three = _grads(4, 4096, 12, 3.0, 3, 11, fold_terms=3)
    one = _grads(4, 4096, 12, 3.0, 3, 11, fold_terms=1)
    assert max(one) > 2e-2 > max(three)


def test_e4m3_inputs_move_the_result_beyond_the_tolerances():
    # An FP8 forward (e4m3 q, k, v with a per-tensor scale) changes the
    # attention it computes, not only its rounding: at the bench workload the
    # same fp16-P arithmetic on the e4m3 inputs is ~10x outside the out and
    # lse tolerances of the oracle on the bf16 inputs. Such a path is checked
    # against the oracle on its dequantized inputs instead.
    import torch

    def e4m3(x):
        s = np.float32(448.0) / np.float32(np.abs(x).max())
        q = torch.from_numpy((np.asarray(x, np.float32) * s).astype(np.float32))
        return q.to(torch.float8_e4m3fn).to(torch.float32).numpy() / s

    Q, K, V = _head(16, 1024, 12, 1.0, 0, 0)
    O, lse, _ = orc.head_forward(Q, K, V, 0.125)
    Qq, Kq, Vq = e4m3(Q), e4m3(K), e4m3(V)
    out, lse_m = kernel_forward_model(Qq, Kq, Vq, 0.125, "f16")
    assert np.max(np.abs(out.astype(np.float64) - O)) > 5e-2
    assert np.max(np.abs(lse_m - lse)) > 2e-2
    # Against the oracle on the dequantized inputs the same arithmetic is
    # inside the tolerances again.
    Oq, lseq, _ = orc.head_forward(Qq.astype(np.float64), Kq.astype(np.float64), Vq.astype(np.float64), 0.125)
    ok, err, _ = out_error_ok(out.astype(np.float64), Oq)
    assert ok, err
    assert np.max(np.abs(lse_m - lseq)) <= LSE_TOL


def test_fp8_forward_model_rounds_faithfully_on_peaked_rows():
    # The FP8 forward's arithmetic (exact e4m3 logits, fp16 P and V) on the
    # dequantised stress inputs, head (0, 8): one output element near 4 lies
    # about 2e-3 from the exact value in fp32 and rounds to the far bf16
    # neighbour, so correct rounding fails while faithful rounding (either
    # enclosing bf16 value) holds; lse stays far inside 1e-3.
    from oracle import fp8 as ofp8
    from .test_parity_gpu import out_error_ok, out_error_ok_faithful

    qkv, _ = make_inputs(4, 4096, 12, 64, seed=0, qk_std=3.0)
    bits, dq = ofp8.quantize_qkv(qkv.float().numpy())
    deq = ofp8.dequantize_qkv(bits, dq)
    Q, K, V = (deq[0, :, s, 8] for s in range(3))
    O, lse, _ = orc.head_forward(Q, K, V, 0.125)
    out, lse_m = kernel_forward_model(Q, K, V, 0.125, "f16")
    assert not out_error_ok(out.astype(np.float64), O)[0]
    assert out_error_ok_faithful(out.astype(np.float64), O)[0]
    assert np.max(np.abs(lse_m - lse)) <= LSE_TOL
