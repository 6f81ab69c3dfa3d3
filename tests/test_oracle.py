"""The fp64 oracle against what the definition fixes (CPU only).

Each pin in ``tests/pins.py`` runs against the oracle and must pass. The
same pins then run against plausible broken copies (a shifted mask, a
dropped scale, a transposed operand, a wrong sign, a dropped Jacobian term,
a base-2 LSE). At least one pin must reject each copy, which shows that the
pins could catch such a mistake in the oracle itself.
"""

import json
import os

import numpy as np
import pytest

from oracle import brute
from oracle import oracle as orc

from . import pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "causal_T3_closed_form.json")


def ora_fwd(qkv, scale):
    return orc.attention_forward(qkv, scale)


def ora_fwdbwd(qkv, dout, scale):
    return orc.attention_forward_backward(qkv, dout, scale)


def ora_probs(Q, K, scale):
    return orc.causal_softmax(orc.causal_scores(Q, K, scale))[0]


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_golden_closed_form(golden):
    pins.pin_closed_form_fixture(ora_fwdbwd, golden)


def test_row_sums_and_support():
    pins.pin_row_sums_and_support(ora_probs)


def test_query_zero_returns_v0_exactly():
    pins.pin_query_zero(ora_fwd)


def test_zero_queries_give_prefix_mean():
    pins.pin_zero_queries_prefix_mean(ora_fwd)


def test_single_token_closed_form():
    pins.pin_single_token(ora_fwdbwd)


def test_key_shift_invariance():
    pins.pin_key_shift(ora_fwdbwd)


def test_finite_differences():
    pins.pin_finite_differences(ora_fwdbwd)


def test_delta_shortcut_matches_jacobian_row_term():
    """sum_k P_ik dP_ik == dO_i . O_i: the quantity the GPU backward uses."""
    r = np.random.default_rng(7)
    B, T, H, D = 2, 19, 3, 8
    qkv = r.standard_normal((B, T, 3, H, D))
    dout = r.standard_normal((B, T, H, D))
    out, _ = orc.attention_forward(qkv, 0.125)
    delta = orc.delta_rowsum(out, dout)
    for b in range(B):
        for h in range(H):
            _, _, P = orc.head_forward(qkv[b, :, 0, h], qkv[b, :, 1, h], qkv[b, :, 2, h], 0.125)
            dP = dout[b, :, h] @ qkv[b, :, 2, h].T
            row = np.sum(P * dP, axis=1)
            assert np.allclose(row, delta[b, h], rtol=0, atol=1e-12)


@pytest.mark.parametrize("T,D,H", [(1, 3, 1), (5, 4, 2), (16, 8, 2)])
def test_matches_pure_python_loops(T, D, H):
    r = np.random.default_rng(100 + T)
    qkv = r.standard_normal((1, T, 3, H, D))
    dout = r.standard_normal((1, T, H, D))
    scale = 1.0 / np.sqrt(D)
    out, lse, dqkv = ora_fwdbwd(qkv, dout, scale)
    for h in range(H):
        q, k, v = (qkv[0, :, s, h].tolist() for s in range(3))
        do = dout[0, :, h].tolist()
        o_b, lse_b, _ = brute.forward(q, k, v, scale)
        dq_b, dk_b, dv_b = brute.backward(q, k, v, do, scale)
        assert np.allclose(out[0, :, h], o_b, rtol=0, atol=1e-12)
        assert np.allclose(lse[0, h], lse_b, rtol=0, atol=1e-12)
        assert np.allclose(dqkv[0, :, 0, h], dq_b, rtol=0, atol=1e-12)
        assert np.allclose(dqkv[0, :, 1, h], dk_b, rtol=0, atol=1e-12)
        assert np.allclose(dqkv[0, :, 2, h], dv_b, rtol=0, atol=1e-12)


def test_brute_closed_form(golden):
    """The loop oracle also reproduces the hand-worked fixture."""

    def fwdbwd(qkv, dout, scale):
        B, T, _, H, D = qkv.shape
        q, k, v = (qkv[0, :, s, 0].tolist() for s in range(3))
        do = dout[0, :, 0].tolist()
        o, lse, _ = brute.forward(q, k, v, scale)
        dq, dk, dv = brute.backward(q, k, v, do, scale)
        dqkv = np.stack([np.array(dq), np.array(dk), np.array(dv)], axis=1)[None, :, :, None]
        return np.array(o)[None, :, None], np.array(lse)[None, None], dqkv

    pins.pin_closed_form_fixture(fwdbwd, golden)


def test_library_crosscheck_torch_sdpa_fp64():
    """At the small GPT-2 shape (B=1, T=128, H=12, D=64) the oracle agrees with
    torch's fp64 CPU causal scaled-dot-product attention and its autograd."""
    import torch
    import torch.nn.functional as F

    from causal_self_attention_flashattention_b200.workload import make_inputs

    qkv_bf, dout_bf = make_inputs(1, 128, 12, 64, seed=0)
    qkv = qkv_bf.double()
    dout = dout_bf.double()
    out, lse, dqkv = ora_fwdbwd(qkv.numpy(), dout.numpy(), 0.125)

    x = qkv.clone().requires_grad_(True)
    q, k, v = (x[:, :, s].transpose(1, 2) for s in range(3))  # (B,H,T,D)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=0.125)
    o = o.transpose(1, 2)
    (o * dout).sum().backward()
    assert np.allclose(out, o.detach().numpy(), rtol=0, atol=1e-10)
    assert np.allclose(dqkv, x.grad.numpy(), rtol=0, atol=1e-10)
    s = 0.125 * torch.einsum("bihd,bjhd->bhij", qkv[:, :, 0], qkv[:, :, 1])
    s = s.masked_fill(torch.triu(torch.ones(128, 128, dtype=torch.bool), 1), float("-inf"))
    assert np.allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-10)


def test_worker_processes_give_identical_results():
    r = np.random.default_rng(8)
    qkv = r.standard_normal((2, 40, 3, 3, 8))
    dout = r.standard_normal((2, 40, 3, 8))
    a = orc.attention_forward_backward(qkv, dout, 0.2)
    b = orc.attention_forward_backward(qkv, dout, 0.2, processes=2)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# ---------------------------------------------------------------------------
# Planted mistakes: each broken copy must be rejected by at least one pin.
# ---------------------------------------------------------------------------

def _mutant(kind):
    """A copy of the oracle with one plausible mistake planted in it."""

    def scores(Q, K, scale):
        T = Q.shape[0]
        s = (Q @ K.T) * (1.0 if kind == "no_scale" else scale)
        if kind == "strict_mask":      # diagonal hidden, row 0 gets key 1 instead
            mask = np.tril(np.ones((T, T), dtype=bool), k=-1)
            mask[0, min(1, T - 1)] = True
            s = np.where(mask, s, -np.inf)
        elif kind == "anti_causal":
            s[np.tril_indices(T, k=-1)] = -np.inf
        else:
            s[np.triu_indices(T, k=1)] = -np.inf
        return s

    def softmax(s):
        m = np.max(s, axis=1)
        if kind == "lse_base2":
            lse = m + np.log2(np.sum(np.exp(s - m[:, None]), axis=1))
            P = np.exp(s - m[:, None])
            P /= P.sum(axis=1, keepdims=True)
            return P, lse
        lse = m + np.log(np.sum(np.exp(s - m[:, None]), axis=1))
        return np.exp(s - lse[:, None]), lse

    def head(Q, K, V, dO, scale):
        P, lse = softmax(scores(Q, K, scale))
        O = P @ V
        dV = (dO.T @ P).T if kind != "dv_transposed" else P @ dO
        dP = dO @ V.T
        row = np.sum(P * dP, axis=1)
        if kind == "drop_row_term":
            dS = P * dP
        elif kind == "sign_flip":
            dS = P * (row[:, None] - dP)
        else:
            dS = P * (dP - row[:, None])
        dQ = scale * (dS @ K)
        dK = scale * ((dS if kind == "dk_transposed" else dS.T) @ Q)
        return O, lse, dQ, dK, dV

    def fwdbwd(qkv, dout, scale):
        qkv = np.asarray(qkv, dtype=np.float64)
        B, T, _, H, D = qkv.shape
        out = np.empty((B, T, H, D))
        lse = np.empty((B, H, T))
        g = np.empty((B, T, 3, H, D))
        for b in range(B):
            for h in range(H):
                O, l, dQ, dK, dV = head(qkv[b, :, 0, h], qkv[b, :, 1, h], qkv[b, :, 2, h],
                                        np.asarray(dout, dtype=np.float64)[b, :, h], scale)
                out[b, :, h], lse[b, h] = O, l
                g[b, :, 0, h], g[b, :, 1, h], g[b, :, 2, h] = dQ, dK, dV
        return out, lse, g

    def fwd(qkv, scale):
        B, T, _, H, D = np.shape(qkv)
        o, l, _ = fwdbwd(qkv, np.zeros((B, T, H, D)), scale)
        return o, l

    def probs(Q, K, scale):
        return softmax(scores(Q, K, scale))[0]

    return fwd, fwdbwd, probs


MUTANTS = ["no_scale", "strict_mask", "anti_causal", "lse_base2", "dv_transposed",
           "drop_row_term", "sign_flip", "dk_transposed"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_pins_reject_planted_mistake(kind, golden):
    fwd, fwdbwd, probs = _mutant(kind)
    checks = [
        lambda: pins.pin_closed_form_fixture(fwdbwd, golden),
        lambda: pins.pin_row_sums_and_support(probs),
        lambda: pins.pin_query_zero(fwd),
        lambda: pins.pin_zero_queries_prefix_mean(fwd),
        lambda: pins.pin_single_token(fwdbwd),
        lambda: pins.pin_key_shift(fwdbwd),
        lambda: pins.pin_finite_differences(fwdbwd),
    ]
    failed = 0
    for c in checks:
        try:
            with np.errstate(all="ignore"):
                c()
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake {kind!r}"


def test_unmodified_copy_passes_every_pin(golden):
    """The mutant scaffold with no mistake planted passes all pins, so the
    rejections above come from the planted mistakes and not the scaffold."""
    fwd, fwdbwd, probs = _mutant("none")
    pins.pin_closed_form_fixture(fwdbwd, golden)
    pins.pin_row_sums_and_support(probs)
    pins.pin_query_zero(fwd)
    pins.pin_zero_queries_prefix_mean(fwd)
    pins.pin_single_token(fwdbwd)
    pins.pin_key_shift(fwdbwd)
    pins.pin_finite_differences(fwdbwd)
