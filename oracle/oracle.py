"""fp64 CPU oracle for causal multi-head self-attention, forward and backward.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it. It shares no code with the CUDA library.

What it computes
----------------
The operation is the attention step inside every block of GPT-2 (124M): 12
layers of width 768 ("Let's reproduce GPT-2 (124M)" video summary page,
closing summary paragraph). Flash attention computes that attention without
ever storing the full T x T attention matrix (same page, glossary table, row
"flash attention"; the "Andrej Karpathy - Lets reproduce GPT 2 124M" video
description, chapter 02:00:18 "flash attention"). Flash attention therefore
reaches the same numbers as the plain definition, up to rounding order. This
oracle is the plain definition, written out in fp64 with the full matrix:

    s_ij  = scale * q_i . k_j        for j <= i,   -inf for j > i
    lse_i = log sum_j exp(s_ij)      (natural log, scaled logits)
    P_ij  = exp(s_ij - lse_i)
    O     = P V

and its analytic gradients, for an upstream gradient dO:

    dV    = P^T dO
    dP    = dO V^T
    dS_ij = P_ij * (dP_ij - sum_k P_ik dP_ik)      (softmax Jacobian, row by row)
    dQ    = scale * dS K
    dK    = scale * dS^T Q

The causal mask (key j visible to query i iff j <= i) follows from GPT-2 being
a left-to-right language model (video description, chapters 00:31:00 "logits"
and 00:37:02 "generation loop"). The pages print neither the mask, the scale
nor the logsumexp convention; the readings taken are: diagonal included,
scale passed explicitly (1/sqrt(D) for GPT-2), natural-log LSE of the scaled
logits.

Layouts (the GPT-2 ``c_attn`` output split into heads):
    qkv   (B, T, 3, H, D)   slot 0 = q, 1 = k, 2 = v
    out   (B, T, H, D)
    lse   (B, H, T)
    dout  (B, T, H, D)
    dqkv  (B, T, 3, H, D)

Every array is converted to float64 on entry. bf16 inputs must be upcast
exactly by the caller (``torch.Tensor.double()`` does that).
"""

from __future__ import annotations

import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

__all__ = [
    "causal_scores",
    "causal_softmax",
    "head_forward",
    "head_backward",
    "attention_forward",
    "attention_backward",
    "attention_forward_backward",
    "delta_rowsum",
]


def causal_scores(Q: np.ndarray, K: np.ndarray, scale: float) -> np.ndarray:
    """Scaled logits s = scale * Q K^T with -inf wherever key j > query i.

    Q, K: (T, D). Returns a (T, T) float64 array.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    T = Q.shape[0]
    s = float(scale) * (Q @ K.T)
    future = np.triu(np.ones((T, T), dtype=bool), k=1)  # j > i
    s[future] = -np.inf
    return s


def causal_softmax(s: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Row-wise softmax of masked logits and the row logsumexp.

    Uses the textbook stabilised form lse_i = m_i + log sum_j exp(s_ij - m_i),
    m_i = max_j s_ij. Every row has at least its diagonal entry visible, so
    m_i is finite. Returns (P, lse) with P (T, T) and lse (T,).
    """
    m = np.max(s, axis=1)
    lse = m + np.log(np.sum(np.exp(s - m[:, None]), axis=1))
    P = np.exp(s - lse[:, None])
    return P, lse


def head_forward(Q, K, V, scale):
    """One head's forward pass: returns (O, lse, P)."""
    s = causal_scores(Q, K, scale)
    P, lse = causal_softmax(s)
    O = P @ np.asarray(V, dtype=np.float64)
    return O, lse, P


def head_backward(Q, K, V, dO, scale):
    """One head's analytic gradients (dQ, dK, dV), via the explicit Jacobian.

    The softmax Jacobian is applied as dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik).
    The shortcut sum_k P_ik dP_ik = dO_i . O_i is *not* used here. The
    identity between the two is checked separately (``delta_rowsum``).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    _, _, P = head_forward(Q, K, V, scale)
    dV = P.T @ dO
    dP = dO @ V.T
    row = np.sum(P * dP, axis=1)
    dS = P * (dP - row[:, None])
    dQ = float(scale) * (dS @ K)
    dK = float(scale) * (dS.T @ Q)
    return dQ, dK, dV


def delta_rowsum(out, dout) -> np.ndarray:
    """Delta[b, h, t] = sum_d dout[b, t, h, d] * out[b, t, h, d].

    This is the per-row quantity a flash-attention backward uses in place of
    sum_k P_ik dP_ik. out and dout are (B, T, H, D); the result is (B, H, T).
    """
    o = np.asarray(out, dtype=np.float64)
    g = np.asarray(dout, dtype=np.float64)
    return np.einsum("bthd,bthd->bht", o, g)


# ---------------------------------------------------------------------------
# Whole-tensor drivers: loop (optionally in worker processes) over (b, h).
# ---------------------------------------------------------------------------

def _split(qkv):
    qkv = np.asarray(qkv, dtype=np.float64)
    if qkv.ndim != 5 or qkv.shape[2] != 3:
        raise ValueError(f"qkv must be (B, T, 3, H, D), got {qkv.shape}")
    return qkv


def _fwd_task(args):
    Q, K, V, scale = args
    O, lse, _ = head_forward(Q, K, V, scale)
    return O, lse


def _fwd_bwd_task(args):
    Q, K, V, dO, scale = args
    O, lse, _ = head_forward(Q, K, V, scale)
    dQ, dK, dV = head_backward(Q, K, V, dO, scale)
    return O, lse, dQ, dK, dV


def _worker_init():
    # One BLAS thread per worker process: the parallelism is over heads.
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"


def _map(fn, tasks, processes):
    if processes is None or processes <= 1 or len(tasks) <= 1:
        return [fn(t) for t in tasks]
    import multiprocessing as mp

    ctx = mp.get_context("spawn")  # never fork a process that may hold a CUDA context
    with ProcessPoolExecutor(max_workers=processes, mp_context=ctx,
                             initializer=_worker_init) as ex:
        return list(ex.map(fn, tasks, chunksize=max(1, len(tasks) // (4 * processes))))


def attention_forward(qkv, scale, processes=None):
    """Forward over all heads. qkv (B,T,3,H,D) -> (out (B,T,H,D), lse (B,H,T))."""
    qkv = _split(qkv)
    B, T, _, H, D = qkv.shape
    tasks = [(qkv[b, :, 0, h], qkv[b, :, 1, h], qkv[b, :, 2, h], scale)
             for b in range(B) for h in range(H)]
    res = _map(_fwd_task, tasks, processes)
    out = np.empty((B, T, H, D))
    lse = np.empty((B, H, T))
    for idx, (O, l) in enumerate(res):
        b, h = divmod(idx, H)
        out[b, :, h] = O
        lse[b, h] = l
    return out, lse


def attention_forward_backward(qkv, dout, scale, processes=None):
    """Forward and backward over all heads.

    Returns (out (B,T,H,D), lse (B,H,T), dqkv (B,T,3,H,D)).
    """
    qkv = _split(qkv)
    dout = np.asarray(dout, dtype=np.float64)
    B, T, _, H, D = qkv.shape
    if dout.shape != (B, T, H, D):
        raise ValueError(f"dout must be {(B, T, H, D)}, got {dout.shape}")
    tasks = [(qkv[b, :, 0, h], qkv[b, :, 1, h], qkv[b, :, 2, h], dout[b, :, h], scale)
             for b in range(B) for h in range(H)]
    res = _map(_fwd_bwd_task, tasks, processes)
    out = np.empty((B, T, H, D))
    lse = np.empty((B, H, T))
    dqkv = np.empty((B, T, 3, H, D))
    for idx, (O, l, dQ, dK, dV) in enumerate(res):
        b, h = divmod(idx, H)
        out[b, :, h] = O
        lse[b, h] = l
        dqkv[b, :, 0, h] = dQ
        dqkv[b, :, 1, h] = dK
        dqkv[b, :, 2, h] = dV
    return out, lse, dqkv


def attention_backward(qkv, dout, scale, processes=None):
    """Backward over all heads: returns dqkv (B,T,3,H,D)."""
    return attention_forward_backward(qkv, dout, scale, processes)[2]
