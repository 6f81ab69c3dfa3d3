"""gpt2_attn_bwd_noalloc: the backward for callers that cannot allocate.

Some callers cannot call cudaMalloc: a plugin handed only its input and
output buffers by a host application that owns all device memory, or a
program that reserves the GPU's memory at start-up and may not allocate (or
take cudaMalloc's implicit synchronisation) afterwards. For them the library
keeps the backward's Delta scratch in a fixed static device array instead of
a caller workspace. These tests check that entry point through the C ABI
against the workspace-based gpt2_attn_bwd, on two calls in a row, and that
shapes beyond the fixed scratch are refused.

This file is collected last so that a run stopping at its first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from causal_self_attention_flashattention_b200 import ops
from causal_self_attention_flashattention_b200.workload import make_inputs

GRAD_TOL = 2e-2  # relative Frobenius bound used for dq, dk, dv everywhere
MAX_DELTA = 1 << 20


def rel_fro(g, o):
    g = g.double().cpu().numpy()
    o = o.double().cpu().numpy()
    return float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30))


def test_rejects_shapes_beyond_the_fixed_scratch():
    """B*H*T above 2^20 is refused before any CUDA call (runs without a GPU)."""
    p = 0x10000  # aligned, never dereferenced: the call fails its checks first
    lib = ops.lib()
    # 2 * 513 * 1024 = 1,050,624 > 2^20
    assert lib.gpt2_attn_bwd_noalloc(p, p, p, p, p, 2, 1024, 513, 64, 0.125, None) == ops.GA_ERR_WORKSPACE
    assert lib.gpt2_attn_bwd_noalloc(p, p, p, p, p, 1, 1024, 12, 128, 0.125, None) == ops.GA_ERR_UNSUPPORTED
    assert lib.gpt2_attn_bwd_noalloc(None, p, p, p, p, 1, 1024, 12, 64, 0.125, None) == ops.GA_ERR_INVALID_ARG
    assert lib.gpt2_attn_bwd_noalloc(p, p, p, p, p + 8, 1, 1024, 12, 64, 0.125, None) == ops.GA_ERR_ALIGNMENT


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_on_two_calls(cuda_device):
    """Two calls in a row through the C ABI, the larger B*H*T first, so that a
    read of a Delta entry left over from the earlier call would show. Both
    entry points run the same deterministic dQ and dK/dV kernels on the same
    Delta, so their dqkv must agree bit for bit; one of them is also compared
    with the oracle."""
    from oracle import oracle as orc

    cases = [(1, 1000, 4, 22), (2, 512, 3, 21)]     # B*H*T = 4000, then 3072
    prepared = []
    for B, T, H, seed in cases:
        assert B * H * T <= MAX_DELTA
        qkv_bf, dout_bf = make_inputs(B, T, H, 64, seed=seed)
        qkv, dout = qkv_bf.cuda(), dout_bf.cuda()
        out, lse = ops.attn_fwd(qkv)
        ref = ops.attn_bwd(qkv, out, dout, lse)           # workspace-based entry point
        got = torch.full_like(qkv, float("nan"))
        prepared.append((qkv, out, dout, lse, ref, got, (B, T, H), qkv_bf, dout_bf))
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    for qkv, out, dout, lse, ref, got, (B, T, H), _, _ in prepared:  # two calls in a row
        st = ops.lib().gpt2_attn_bwd_noalloc(
            qkv.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(), got.data_ptr(),
            B, T, H, 64, ctypes.c_float(0.125), ctypes.c_void_p(stream.cuda_stream))
        assert st == ops.GA_OK, ops.status_string(st)
    status, word = ops.last_device_status()
    assert status == ops.GA_OK, (status, hex(word))

    for qkv, out, dout, lse, ref, got, _, _, _ in prepared:
        assert not torch.isnan(got).any()
        assert torch.equal(got, ref)

    # The second (smaller) case against the fp64 oracle as well.
    _, _, _, _, _, got, _, qkv_bf, dout_bf = prepared[1]
    _, _, dqkv_o = orc.attention_forward_backward(qkv_bf.double().numpy(),
                                                  dout_bf.double().numpy(), 0.125)
    for s in range(3):
        assert rel_fro(got[:, :, s], torch.from_numpy(dqkv_o[:, :, s])) <= GRAD_TOL
