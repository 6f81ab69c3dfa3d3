"""The device-side failure path, made to run on purpose without a fault.

Every wait in the library's kernels is bounded. When a limit passes, the
waiting thread records its site in the device status word and raises its
block's abort flag, the block's other roles wind down instead of waiting out
their own limits, tensor memory is freed, and the kernel returns. These tests
drive that path through gpt2_attn_selftest_wait_timeout (a barrier nothing
completes, with a short limit) and check what the host sees afterwards:
GA_ERR_TIMEOUT with the site, then a context that still computes correctly.
"""

import time

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from causal_self_attention_flashattention_b200.workload import make_inputs

pytestmark = pytest.mark.gpu

SITE_SELFTEST_WAIT = 0x501


@pytest.fixture(scope="module")
def ops(cuda_device):
    from causal_self_attention_flashattention_b200 import ops as _ops

    return _ops


def test_selftest_rejects_bad_limits(ops):
    assert ops.lib().gpt2_attn_selftest_wait_timeout(0, None) == ops.GA_ERR_INVALID_ARG
    assert ops.lib().gpt2_attn_selftest_wait_timeout(2_000_000_000, None) == ops.GA_ERR_INVALID_ARG


@pytest.mark.parametrize("limit_ms", [5, 50])
def test_bounded_wait_times_out_and_reports_its_site(ops, limit_ms):
    assert ops.last_device_status() == (ops.GA_OK, 0)
    stream = torch.cuda.current_stream()
    t0 = time.perf_counter()
    st = ops.lib().gpt2_attn_selftest_wait_timeout(limit_ms * 1_000_000, stream.cuda_stream)
    assert st == ops.GA_OK
    status, word = ops.last_device_status(stream)       # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert status == ops.GA_ERR_TIMEOUT, (status, hex(word))
    assert word >> 32 == SITE_SELFTEST_WAIT, hex(word)  # the short wait, not the peer's
    assert word & 0xFFFFFFFF == 0                        # block 0
    # The peer waiter (2 s limit) wound down on the abort flag: the kernel
    # ended a little after the short limit, not after 2 s.
    assert limit_ms * 1e-3 <= elapsed < 1.0, elapsed
    # Reading the word cleared it.
    assert ops.last_device_status() == (ops.GA_OK, 0)


def test_context_usable_after_a_timeout(ops):
    st = ops.lib().gpt2_attn_selftest_wait_timeout(2_000_000, None)
    assert st == ops.GA_OK
    status, _ = ops.last_device_status()
    assert status == ops.GA_ERR_TIMEOUT
    B, T, H = 2, 300, 3
    qkv_bf, dout_bf = make_inputs(B, T, H, 64, seed=77)
    qkv, dout = qkv_bf.cuda(), dout_bf.cuda()
    out, lse = ops.attn_fwd(qkv)
    dqkv = ops.attn_bwd(qkv, out, dout, lse)
    assert ops.last_device_status() == (ops.GA_OK, 0)
    out_o, lse_o, dqkv_o = orc.attention_forward_backward(
        qkv_bf.double().numpy(), dout_bf.double().numpy(), 0.125)
    assert np.max(np.abs(out.cpu().double().numpy() - out_o)) <= 1e-2
    assert np.max(np.abs(lse.cpu().double().numpy() - lse_o)) <= 1e-3
    g = dqkv.cpu().double().numpy()
    for s in range(3):
        rel = np.linalg.norm(g[:, :, s] - dqkv_o[:, :, s]) / np.linalg.norm(dqkv_o[:, :, s])
        assert rel <= 2e-2
