"""The fp16-v inference path: c_attn writing the v slot in fp16
(gpt2_attn_qkv_proj_v16) and the forward reading it without conversion
(gpt2_attn_fwd_v16), through the C ABI.

The bf16 forward converts every V tile to fp16 in shared memory (round to
nearest) before its P V product, and otherwise runs the same arithmetic as
the fp16-v forward. So for a v that both formats hold exactly, the two
forwards must agree bit for bit; that pins the fp16-v kernel to the bf16 one,
whose parity with the oracle the other GPU tests establish. The fp16 v slot
of c_attn is checked against the fp64 linear oracle with the fp16 rounding
margin, and the chain c_attn -> attention against the attention oracle run
on the fp16 v the GPU saw.
"""

import numpy as np
import pytest
import torch

from oracle import linear as lin
from oracle import oracle as orc
from causal_self_attention_flashattention_b200.workload import (WORKLOADS, make_inputs,
                                                               make_linear_inputs)

from .test_parity_gpu import LSE_TOL, out_error_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops(cuda_device):
    from causal_self_attention_flashattention_b200 import ops as _ops

    return _ops


def with_fp16_v(qkv: torch.Tensor) -> torch.Tensor:
    """The same q, k and v values with the v slot stored as fp16 bits."""
    q16 = qkv.clone()
    q16[:, :, 2] = qkv[:, :, 2].to(torch.float16).view(torch.bfloat16)
    return q16


@pytest.mark.parametrize("B,T,H,qk_std", [
    (1, 1, 1, 1.0),
    (2, 300, 3, 1.0),          # ragged last tile, odd number of query tiles
    (1, 1000, 2, 3.0),         # peaked rows
    (16, 1024, 12, 1.0),       # the bench workload
])
def test_fwd_v16_bit_identical_to_bf16_forward(ops, B, T, H, qk_std):
    qkv_bf, _ = make_inputs(B, T, H, 64, seed=60 + T, qk_std=qk_std)
    qkv = qkv_bf.cuda()
    # N(0, 1) bf16 values lie inside fp16's range: the conversion is exact
    # except for fp16 subnormals, which both paths round the same way.
    q16 = with_fp16_v(qkv)
    out_a, lse_a = ops.attn_fwd(qkv)
    out_b, lse_b = ops.attn_fwd_v16(q16)
    assert ops.last_device_status() == (ops.GA_OK, 0)
    assert torch.equal(out_a, out_b)
    assert torch.equal(lse_a, lse_b)


def test_qkv_proj_v16_slots(ops):
    """q and k slots equal the bf16 layer's; the v slot is the fp16 rounding
    of the same fp32 result: |v16 - y| <= 2^-11 |y| + 2^-15 S (fp16 half
    spacing doubled as the margin, plus the fp32 accumulation bound)."""
    B, T, H = 3, 257, 12
    C = 64 * H
    x, w, b = make_linear_inputs(B, T, C, 3 * C, seed=61)
    a = ops.qkv_proj(x.cuda(), w.cuda(), b.cuda(), H)
    v16 = ops.qkv_proj(x.cuda(), w.cuda(), b.cuda(), H, v_fp16=True)
    assert torch.equal(a[:, :, :2], v16[:, :, :2])
    x64 = x.double().numpy().reshape(-1, C)
    w64 = w.double().numpy()
    ref = lin.linear(x64, w64, b.double().numpy()).reshape(B, T, 3, H, 64)[:, :, 2]
    S = (np.abs(x64) @ np.abs(w64).T).reshape(B, T, 3, H, 64)[:, :, 2]
    got = v16[:, :, 2].view(torch.float16).cpu().double().numpy()
    err = np.abs(got - ref)
    bound = 2.0 ** -11 * np.abs(ref) + 2.0 ** -15 * S
    bad = np.argwhere(err > bound)
    assert bad.size == 0, (bad[:5], err[tuple(bad[0])], bound[tuple(bad[0])])
    assert ops.last_device_status() == (ops.GA_OK, 0)


def test_c_attn_v16_then_attention_matches_oracle(ops):
    """The inference chain on its own output: c_attn with an fp16 v slot,
    then the fp16-v forward, against the oracle on the q, k, v values the GPU
    produced (v read as fp16)."""
    B, T, H = 2, 384, 4
    C = 64 * H
    x, w, b = make_linear_inputs(B, T, C, 3 * C, seed=62)
    qkv = ops.qkv_proj(x.cuda(), w.cuda(), b.cuda(), H, v_fp16=True)
    out, lse = ops.attn_fwd_v16(qkv)
    assert ops.last_device_status() == (ops.GA_OK, 0)
    vals = qkv.cpu().double().numpy()
    vals[:, :, 2] = qkv[:, :, 2].view(torch.float16).cpu().double().numpy()
    out_o, lse_o = orc.attention_forward(vals, 0.125)
    ok, err, _ = out_error_ok(out.cpu().double().numpy(), out_o)
    assert ok, err
    assert np.max(np.abs(lse.cpu().double().numpy() - lse_o)) <= LSE_TOL


def test_fwd_v16_argument_errors(ops):
    qkv = torch.zeros(1, 8, 3, 1, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.AttnError):
        ops.attn_fwd_v16(qkv, scale=0.0)
    lib = ops.lib()
    p = qkv.data_ptr()
    assert lib.gpt2_attn_fwd_v16(None, p, p, 1, 8, 1, 64, 0.125, None) == ops.GA_ERR_INVALID_ARG
    assert lib.gpt2_attn_fwd_v16(p, p + 2, p, 1, 8, 1, 64, 0.125, None) == ops.GA_ERR_ALIGNMENT
    assert lib.gpt2_attn_fwd_v16(p, p, p, 1, 8, 1, 32, 0.125, None) == ops.GA_ERR_UNSUPPORTED
