"""Pure-Python triple-loop causal attention, for tiny sizes (T <= 16).

TEST INFRASTRUCTURE ONLY: an independent second oracle used to pin
``oracle.oracle``. It uses no NumPy and no matrix routine, only Python floats
(IEEE fp64) and ``math``, and shares no code with either the NumPy oracle or
the CUDA library.

It computes the same definition (causal softmax attention: key j is visible
to query i iff j <= i, logits scaled by ``scale``, natural-log LSE) and the
gradients. Here they come from the chain rule written element by element:
dL/ds_ij = sum_k dL/dP_ik * P_ik * ([j == k] - P_ij).

All inputs are nested lists: q, k, v, do are [T][D].
"""

from __future__ import annotations

import math


def forward(q, k, v, scale):
    """Returns (o [T][D], lse [T], p [T][T]) for one head."""
    T = len(q)
    D = len(q[0])
    p = [[0.0] * T for _ in range(T)]
    o = [[0.0] * D for _ in range(T)]
    lse = [0.0] * T
    for i in range(T):
        logits = []
        for j in range(i + 1):
            acc = 0.0
            for d in range(D):
                acc += q[i][d] * k[j][d]
            logits.append(scale * acc)
        mx = max(logits)
        tot = 0.0
        for x in logits:
            tot += math.exp(x - mx)
        lse[i] = mx + math.log(tot)
        for j in range(i + 1):
            p[i][j] = math.exp(logits[j] - lse[i])
        for d in range(D):
            acc = 0.0
            for j in range(i + 1):
                acc += p[i][j] * v[j][d]
            o[i][d] = acc
    return o, lse, p


def backward(q, k, v, do, scale):
    """Returns (dq, dk, dv), each [T][D], for the loss L = sum(do * o)."""
    T = len(q)
    D = len(q[0])
    _, _, p = forward(q, k, v, scale)
    dq = [[0.0] * D for _ in range(T)]
    dk = [[0.0] * D for _ in range(T)]
    dv = [[0.0] * D for _ in range(T)]
    for i in range(T):
        # dL/dP_ij = do_i . v_j
        gp = [0.0] * T
        for j in range(i + 1):
            acc = 0.0
            for d in range(D):
                acc += do[i][d] * v[j][d]
            gp[j] = acc
            for d in range(D):
                dv[j][d] += p[i][j] * do[i][d]
        # chain rule through the softmax of row i
        for j in range(i + 1):
            gs = 0.0
            for kk in range(i + 1):
                jac = p[i][kk] * ((1.0 if j == kk else 0.0) - p[i][j])
                gs += gp[kk] * jac
            for d in range(D):
                dq[i][d] += scale * gs * k[j][d]
                dk[j][d] += scale * gs * q[i][d]
    return dq, dk, dv
