"""The Python binding's argument checks, which run before any CUDA call: wrong
rank, device or shape is refused with an exception naming the argument."""

import pytest
import torch

from causal_self_attention_flashattention_b200 import ops


def _qkv(B=1, T=8, H=2, D=64, device="cpu", dtype=torch.bfloat16):
    return torch.zeros(B, T, 3, H, D, dtype=dtype, device=device)


def test_exports_match_the_loaded_library():
    for name in ops.EXPORTED_SYMBOLS:
        assert hasattr(ops.lib(), name), name


@pytest.mark.parametrize("bad", [
    torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16),        # rank 4
    torch.zeros(1, 8, 2, 2, 64, dtype=torch.bfloat16),     # slot dimension 2, not 3
])
def test_forward_refuses_a_non_packed_layout(bad):
    with pytest.raises(ValueError, match="qkv must be"):
        ops.attn_fwd(bad)


def test_forward_refuses_host_tensors():
    with pytest.raises(ValueError, match="qkv must be a CUDA tensor"):
        ops.attn_fwd(_qkv())


def test_backward_and_decode_refuse_host_tensors():
    qkv = _qkv()
    out = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        ops.attn_bwd(qkv, out, out, lse)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        ops.attn_decode(qkv, 3)


def test_default_scale_is_inverse_sqrt_head_dim():
    assert ops.default_scale(64) == 0.125
    assert ops.default_scale(16) == 0.25


def test_status_errors_carry_the_entry_point_name():
    err = ops.AttnError(ops.GA_ERR_ALIGNMENT, "gpt2_attn_fwd")
    assert "gpt2_attn_fwd" in str(err) and "GA_ERR_ALIGNMENT" in str(err)
    assert err.status == ops.GA_ERR_ALIGNMENT
