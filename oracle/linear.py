"""fp64 CPU oracle for the two dense layers around attention in a GPT-2 block.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it. It shares no code with the CUDA library.

What it computes
----------------
Attention in a GPT-2 block sits between two linear layers of the block's
``nn.Module`` ("Andrej Karpathy - Lets reproduce GPT 2 124M" video
description, chapter 00:13:47, section 1: implementing GPT-2 as an
``nn.Module``; "Comment recréer GPT2 en 4 heures ?", section 5: the theory of
attention matches the practice, with the blocks rearranged for PyTorch):

    c_attn:  qkv = x W_attn^T + b_attn     x (M, C) -> qkv (M, 3C)
    c_proj:  y   = out W_proj^T + b_proj   out (M, C) -> y (M, C)

with M = B*T rows and the weights stored the way ``torch.nn.Linear`` stores
them, (out_features, in_features). The pages give the layer names only
through the model's code structure; the readings taken are the plain ones:
c_attn maps width C to 3C, and its output row, split into three blocks of C
and each block into H heads of D, is the packed (B, T, 3, H, D) q, k, v the
attention reads; c_proj maps the attention output (B, T, H, D) = (M, C) back
to width C. Both add their bias.

Every array is converted to float64 on entry; bf16 inputs must be upcast
exactly by the caller (``torch.Tensor.double()`` does that).
"""

from __future__ import annotations

import numpy as np

__all__ = ["linear", "qkv_projection", "output_projection"]


def linear(x, w, b):
    """y = x w^T + b in fp64. x (M, K), w (N, K), b (N,) -> y (M, N)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if x.ndim != 2 or w.ndim != 2 or b.ndim != 1:
        raise ValueError("x (M, K), w (N, K), b (N,) expected")
    if w.shape[1] != x.shape[1] or b.shape[0] != w.shape[0]:
        raise ValueError(f"shape mismatch: x {x.shape}, w {w.shape}, b {b.shape}")
    return x @ w.T + b


def qkv_projection(x, w_attn, b_attn, H):
    """c_attn: x (B, T, C) -> qkv (B, T, 3, H, D) with D = C / H."""
    x = np.asarray(x, dtype=np.float64)
    B, T, C = x.shape
    if C % H:
        raise ValueError("C must be a multiple of H")
    y = linear(x.reshape(B * T, C), w_attn, b_attn)
    if y.shape[1] != 3 * C:
        raise ValueError("w_attn must have 3C rows")
    return y.reshape(B, T, 3, H, C // H)


def output_projection(out, w_proj, b_proj):
    """c_proj: out (B, T, H, D) -> y (B, T, C) with C = H * D."""
    out = np.asarray(out, dtype=np.float64)
    B, T, H, D = out.shape
    return linear(out.reshape(B * T, H * D), w_proj, b_proj).reshape(B, T, H * D)
