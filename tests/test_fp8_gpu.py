"""GPU parity of the FP8 forward through the C ABI.

The quantiser is integer/byte work after one fp32 multiply per element, so
it must match the CPU quantiser (oracle/fp8.py) bit for bit: the e4m3 bytes
and the three dequantisation multipliers. The FP8 forward computes the
attention of the dequantised inputs; it is compared with the fp64 oracle on
exactly those inputs (dequantised on the CPU): lse max-abs <= 1e-3, out
max-abs <= 1e-2 wherever a bf16 value lies within 1e-2 of the exact output,
and, where none does (|o| >= 4), either of the two bf16 values enclosing the
exact output (faithful rounding). The P V product rounds P to fp16 (relative
2^-11), so an fp32 result near 4 can sit ~2e-3 from the exact value and round
to either neighbour: on the T = 4096 stress workload a float32 model of the
kernel's arithmetic (tests/test_precision_model.py) lands on the far
neighbour in 7 of 48 heads, and the GPU reproduces that model's errors to the
last digit. The bf16 path keeps the stricter correct-rounding rule.
"""

import numpy as np
import pytest
import torch

from oracle import fp8 as ofp8
from oracle import oracle as orc
from causal_self_attention_flashattention_b200.workload import WORKLOADS, make_inputs

from .test_parity_gpu import LSE_TOL, host_cores, out_error_ok_faithful

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops(cuda_device):
    from causal_self_attention_flashattention_b200 import ops as _ops

    return _ops


def run_fp8(ops, qkv_bf, scale=0.125):
    qkv8, scales = ops.fp8_quantize(qkv_bf.cuda())
    out, lse = ops.attn_fwd_fp8(qkv8, scales, scale)
    st, word = ops.last_device_status()
    assert st == ops.GA_OK, (st, hex(word))
    return qkv8.cpu().numpy(), scales.cpu().numpy(), out.cpu(), lse.cpu()


def check(ops, qkv_bf, scale=0.125, processes=None):
    bits_g, scales_g, out_g, lse_g = run_fp8(ops, qkv_bf, scale)
    bits_o, dq_o = ofp8.quantize_qkv(qkv_bf.float().numpy())
    assert np.array_equal(bits_g, bits_o)                     # every byte
    assert np.array_equal(scales_g[:3], dq_o)                 # fp32, bit for bit
    deq = ofp8.dequantize_qkv(bits_o, dq_o)
    out_o, lse_o = orc.attention_forward(deq, scale, processes=processes)
    ok, err, n_floor = out_error_ok_faithful(out_g.double().numpy(), out_o)
    assert ok, (err, n_floor)
    err_lse = float(np.max(np.abs(lse_g.double().numpy() - lse_o)))
    assert err_lse <= LSE_TOL, err_lse
    return err, err_lse


@pytest.mark.parametrize("B,T,H,qk_std", [
    (1, 128, 12, 1.0),
    (1, 1, 1, 1.0),
    (2, 100, 3, 1.0),
    (1, 1000, 2, 1.0),       # eight key tiles, ragged
    (3, 640, 2, 1.0),
    (1, 777, 2, 3.0),        # peaked rows
])
def test_fp8_forward_matches_oracle_on_dequantised_inputs(ops, B, T, H, qk_std):
    qkv_bf, _ = make_inputs(B, T, H, 64, seed=B * 7 + T, qk_std=qk_std)
    check(ops, qkv_bf)


def test_fp8_several_items_per_cta(ops):
    qkv_bf, _ = make_inputs(20, 640, 8, 64, seed=3)
    check(ops, qkv_bf, processes=host_cores())


@pytest.mark.parametrize("name", ["gpt2-124m-b16-t1024", "stress-b4-t4096-qk3"])
def test_fp8_full_size_every_head(ops, name):
    wl = WORKLOADS[name]
    qkv_bf, _ = make_inputs(wl.B, wl.T, wl.H, wl.D, seed=0, qk_std=wl.qk_std)
    procs = host_cores() if wl.T <= 1024 else min(host_cores(), 8)
    check(ops, qkv_bf, wl.scale, processes=procs)


def test_fp8_zero_inputs(ops):
    qkv_bf = torch.zeros(1, 200, 3, 2, 64, dtype=torch.bfloat16)
    bits, scales, out, lse = run_fp8(ops, qkv_bf)
    assert np.all(bits == 0) and np.all(scales[:3] == 1.0)
    assert torch.all(out == 0)
    # All logits 0: lse_i = ln(i + 1).
    assert np.allclose(lse.numpy(), np.log(np.arange(1, 201))[None, None, :], atol=1e-5)


def test_fp8_quantize_rejects_bad_args(ops):
    lib = ops.lib()
    p = 0x10000
    assert lib.gpt2_attn_fp8_quantize(None, p, p, 1, 8, 1, 64, None) == ops.GA_ERR_INVALID_ARG
    assert lib.gpt2_attn_fp8_quantize(p, p, p + 4, 1, 8, 1, 64, None) == ops.GA_ERR_ALIGNMENT
    assert lib.gpt2_attn_fwd_fp8(p, p, p, p, 1, 8, 1, 32, 0.125, None) == ops.GA_ERR_UNSUPPORTED
