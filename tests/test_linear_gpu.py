"""GPU parity of the dense layers around attention (c_attn, c_proj) against
the fp64 oracle (oracle/linear.py), through the C ABI.

Tolerance, derived from the arithmetic: inputs and weights are bf16 (their
products are exact in fp32), the tensor core accumulates the K products in
fp32, the bias is added in fp32 and the result is rounded once to bf16. So
every element obeys
    |y_gpu - y| <= 2^-8 |y| + 2^-15 S,    S = sum_k |x_k| |w_k|,
where 2^-8 |y| is twice the bf16 half-spacing (a rounding margin) and
2^-15 S bounds the fp32 accumulation error with room to spare (a K = 768
worst case is 768 * 2^-24 S ~ 2^-14.4 S; the typical error is sqrt(K) times
smaller). A misplaced tile, a dropped K step, a wrong bias or a transposed
weight moves elements by O(|y|) and fails it at once. The relative Frobenius
error, dominated by the output rounding, must also stay below 4e-3.
"""

import numpy as np
import pytest
import torch

from oracle import linear as lin
from causal_self_attention_flashattention_b200.workload import make_linear_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops(cuda_device):
    from causal_self_attention_flashattention_b200 import ops as _ops

    return _ops


def check(g, x, w, b):
    x64 = x.double().numpy().reshape(-1, x.shape[-1])
    w64 = w.double().numpy()
    ref = lin.linear(x64, w64, b.double().numpy())
    S = np.abs(x64) @ np.abs(w64).T
    g = g.double().numpy().reshape(ref.shape)
    err = np.abs(g - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -15 * S
    bad = np.argwhere(err > bound)
    assert bad.size == 0, (bad[:5], err[tuple(bad[0])], bound[tuple(bad[0])])
    rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    assert rel <= 4e-3, rel
    return float(err.max()), float(rel)


@pytest.mark.parametrize("B,T,H", [
    (1, 100, 2),      # one ragged 128-row tile, C = 128
    (2, 300, 3),      # C = 192: 3C = 576 has a 64-column tail past two 256-column tiles
    (1, 1, 1),        # a single row
    (3, 257, 12),     # the GPT-2 width, ragged rows
])
def test_qkv_and_out_proj_match_oracle(ops, B, T, H):
    C = 64 * H
    x, w, b = make_linear_inputs(B, T, C, 3 * C, seed=B * 100 + T)
    qkv = ops.qkv_proj(x.cuda(), w.cuda(), b.cuda(), H)
    assert qkv.shape == (B, T, 3, H, 64)
    check(qkv.cpu(), x, w, b)
    o, wp, bp = make_linear_inputs(B, T, C, C, seed=B * 100 + T + 1)
    y = ops.out_proj(o.cuda().view(B, T, H, 64), wp.cuda(), bp.cuda())
    check(y.cpu(), o, wp, bp)
    assert ops.last_device_status() == (ops.GA_OK, 0)


def test_full_size_gpt2_124m(ops):
    """B=16, T=1024, C=768 (M = 16384): every element of both layers."""
    B, T, H = 16, 1024, 12
    C = 64 * H
    x, w, b = make_linear_inputs(B, T, C, 3 * C, seed=7)
    qkv = ops.qkv_proj(x.cuda(), w.cuda(), b.cuda(), H)
    check(qkv.cpu(), x, w, b)
    o, wp, bp = make_linear_inputs(B, T, C, C, seed=8)
    y = ops.out_proj(o.cuda().view(B, T, H, 64), wp.cuda(), bp.cuda())
    check(y.cpu(), o, wp, bp)
    assert ops.last_device_status() == (ops.GA_OK, 0)


def test_block_chain_c_attn_attention_c_proj(ops):
    """c_attn writes the packed qkv the attention reads, and c_proj reads the
    attention output as is: the chain against the oracles chained in fp64
    (from the same bf16 tensors the GPU saw at each step)."""
    from oracle import oracle as orc

    B, T, H = 2, 256, 4
    C = 64 * H
    x, w, b = make_linear_inputs(B, T, C, 3 * C, seed=9)
    _, wp, bp = make_linear_inputs(B, T, C, C, seed=10)
    qkv = ops.qkv_proj(x.cuda(), w.cuda(), b.cuda(), H)
    out, _ = ops.attn_fwd(qkv)
    y = ops.out_proj(out, wp.cuda(), bp.cuda())
    check(qkv.cpu(), x, w, b)
    out_o, _ = orc.attention_forward(qkv.cpu().double().numpy(), 0.125)
    assert np.max(np.abs(out.cpu().double().numpy() - out_o)) <= 1e-2
    check(y.cpu(), out.cpu().view(B, T, C), wp, bp)


def test_argument_errors(ops):
    x = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(384, 128, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(384, dtype=torch.bfloat16, device="cuda")
    qkv = torch.empty(1, 4, 3, 2, 64, dtype=torch.bfloat16, device="cuda")
    lib = ops.lib()
    assert lib.gpt2_attn_qkv_proj(x.data_ptr(), w.data_ptr(), b.data_ptr(), qkv.data_ptr(),
                                  1, 4, 2, 32, None) == ops.GA_ERR_UNSUPPORTED
    assert lib.gpt2_attn_qkv_proj(x.data_ptr(), w.data_ptr(), None, qkv.data_ptr(),
                                  1, 4, 2, 64, None) == ops.GA_ERR_INVALID_ARG
    assert lib.gpt2_attn_qkv_proj(x.data_ptr() + 2, w.data_ptr(), b.data_ptr(), qkv.data_ptr(),
                                  1, 4, 2, 64, None) == ops.GA_ERR_ALIGNMENT
