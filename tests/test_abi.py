"""The C ABI: the library loads, exports every declared symbol, and rejects bad
arguments with the documented status before anything reaches a device.

Runs without a GPU: each call here fails argument checking, which happens
before any CUDA call.
"""

import ctypes
import os
import re

import pytest

from causal_self_attention_flashattention_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")

# A pointer value that is 16-byte aligned but never dereferenced (every call
# below fails its checks first).
P = 0x10000
P_MIS = 0x10008


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)
    return [n for n in names if n not in ("defined",)]


def test_library_exports_every_declared_function():
    decl = declared_functions()
    assert "gpt2_attn_fwd" in decl and "gpt2_attn_bwd" in decl
    for name in decl:
        assert hasattr(ops.lib(), name), f"{name} declared in include/ but not exported"
    assert set(ops.EXPORTED_SYMBOLS) <= set(decl)


def test_status_strings_and_version():
    for code in range(8):
        s = ops.status_string(code)
        assert s.startswith("GA_")
    assert "unknown" in ops.status_string(99)
    assert ops.version() >= 100


def fwd(qkv=P, out=P, lse=P, B=1, T=128, H=12, D=64, scale=0.125):
    return ops.lib().gpt2_attn_fwd(qkv, out, lse, B, T, H, D, scale, None)


def bwd(qkv=P, out=P, dout=P, lse=P, dqkv=P, ws=P, ws_bytes=1 << 20,
        B=1, T=128, H=12, D=64, scale=0.125):
    return ops.lib().gpt2_attn_bwd(qkv, out, dout, lse, dqkv, ws, ws_bytes, B, T, H, D, scale, None)


@pytest.mark.parametrize("kw,status", [
    (dict(qkv=None), ops.GA_ERR_INVALID_ARG),
    (dict(out=None), ops.GA_ERR_INVALID_ARG),
    (dict(lse=None), ops.GA_ERR_INVALID_ARG),
    (dict(B=0), ops.GA_ERR_INVALID_ARG),
    (dict(T=-1), ops.GA_ERR_INVALID_ARG),
    (dict(H=0), ops.GA_ERR_INVALID_ARG),
    (dict(D=128), ops.GA_ERR_UNSUPPORTED),
    (dict(D=32), ops.GA_ERR_UNSUPPORTED),
    (dict(scale=0.0), ops.GA_ERR_INVALID_ARG),
    (dict(scale=-1.0), ops.GA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), ops.GA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), ops.GA_ERR_INVALID_ARG),
    (dict(B=1 << 14, T=1 << 14, H=12), ops.GA_ERR_INVALID_ARG),  # >= 2^31 elements
    (dict(qkv=P_MIS), ops.GA_ERR_ALIGNMENT),
    (dict(out=P_MIS), ops.GA_ERR_ALIGNMENT),
    (dict(lse=P + 4), ops.GA_ERR_ALIGNMENT),
])
def test_fwd_rejects(kw, status):
    assert fwd(**kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(dout=None), ops.GA_ERR_INVALID_ARG),
    (dict(dqkv=None), ops.GA_ERR_INVALID_ARG),
    (dict(D=80), ops.GA_ERR_UNSUPPORTED),
    (dict(ws=None), ops.GA_ERR_WORKSPACE),
    (dict(ws_bytes=16), ops.GA_ERR_WORKSPACE),
    (dict(ws=P + 8), ops.GA_ERR_ALIGNMENT),
    (dict(dqkv=P + 2), ops.GA_ERR_ALIGNMENT),
    (dict(scale=0.0), ops.GA_ERR_INVALID_ARG),
])
def test_bwd_rejects(kw, status):
    assert bwd(**kw) == status


def bwd_dq(qkv=P, out=P, dout=P, lse=P, delta=P, dqkv=P, B=1, T=128, H=12, D=64, scale=0.125):
    return ops.lib().gpt2_attn_bwd_dq(qkv, out, dout, lse, delta, dqkv, B, T, H, D, scale, None)


def bwd_dkdv(qkv=P, dout=P, lse=P, delta=P, dqkv=P, B=1, T=128, H=12, D=64, scale=0.125):
    return ops.lib().gpt2_attn_bwd_dkdv(qkv, dout, lse, delta, dqkv, B, T, H, D, scale, None)


@pytest.mark.parametrize("kw,status", [
    (dict(out=None), ops.GA_ERR_INVALID_ARG),
    (dict(delta=None), ops.GA_ERR_INVALID_ARG),
    (dict(qkv=None), ops.GA_ERR_INVALID_ARG),
    (dict(out=P_MIS), ops.GA_ERR_ALIGNMENT),
    (dict(delta=P + 4), ops.GA_ERR_ALIGNMENT),
    (dict(dqkv=P + 2), ops.GA_ERR_ALIGNMENT),
    (dict(D=128), ops.GA_ERR_UNSUPPORTED),
    (dict(T=0), ops.GA_ERR_INVALID_ARG),
    (dict(scale=-0.5), ops.GA_ERR_INVALID_ARG),
])
def test_bwd_dq_rejects(kw, status):
    # The dQ step reads out (for Delta) and writes delta; dK/dV reads delta.
    assert bwd_dq(**kw) == status
    if "out" not in kw:
        assert bwd_dkdv(**kw) == status


def _align256(x):
    return (x + 255) // 256 * 256


def test_workspace_size():
    # The split backward: Delta fp32 (B,H,T), rounded up to 256 bytes.
    assert ops.bwd_workspace_size(16, 1024, 12, 64) == 16 * 12 * 1024 * 4
    assert ops.bwd_workspace_size(1, 5, 1, 64) == 256
    # The fused backward: Delta | dQ sums fp32 (B,H,128*ceil(T/128),D) |
    # counters u32 (B,H,ceil(T/128)), each part rounded up to 256 bytes.
    def layout(B, T, H):
        n = -(-T // 128)
        return (_align256(4 * B * H * T) + _align256(4 * B * H * 128 * n * 64)
                + _align256(4 * B * H * n))
    assert ops.bwd_fused_workspace_size(16, 1024, 12, 64) == layout(16, 1024, 12) == 51_124_224
    assert ops.bwd_fused_workspace_size(1, 5, 1, 64) == layout(1, 5, 1) == 256 + 32768 + 256
    n = ctypes.c_size_t(0)
    assert ops.lib().gpt2_attn_bwd_workspace_size(1, 8, 1, 64, None) == ops.GA_ERR_INVALID_ARG
    assert ops.lib().gpt2_attn_bwd_workspace_size(1, 8, 1, 48, ctypes.byref(n)) == ops.GA_ERR_UNSUPPORTED
    with pytest.raises(ops.AttnError):
        ops.bwd_workspace_size(0, 8, 1, 64)


def test_decode_arguments_rejected_before_launch():
    lib = ops.lib()
    p = 1 << 20  # a 16-byte-aligned fake address: nothing is launched on these paths
    n = ctypes.c_size_t(0)
    assert lib.gpt2_attn_decode_workspace_size(2, 1000, 3, 64, ctypes.byref(n)) == ops.GA_OK
    # partials fp32 [B][H][ceil(T/128)][2 + D]
    assert n.value == 2 * 3 * 8 * 66 * 4
    ws = n.value
    assert lib.gpt2_attn_decode(p, 1000, p, p, p, ws, 2, 1000, 3, 64, 0.125, None) == ops.GA_ERR_INVALID_ARG
    assert lib.gpt2_attn_decode(p, -1, p, p, p, ws, 2, 1000, 3, 64, 0.125, None) == ops.GA_ERR_INVALID_ARG
    assert lib.gpt2_attn_decode(p, 5, p, p, p, ws - 4, 2, 1000, 3, 64, 0.125, None) == ops.GA_ERR_WORKSPACE
    assert lib.gpt2_attn_decode(p, 5, p, p, None, ws, 2, 1000, 3, 64, 0.125, None) == ops.GA_ERR_WORKSPACE
    assert lib.gpt2_attn_decode(p, 5, p, p + 4, p, ws, 2, 1000, 3, 64, 0.125, None) == ops.GA_ERR_ALIGNMENT
    assert lib.gpt2_attn_decode(p, 5, p, p, p, ws, 2, 1000, 3, 32, 0.125, None) == ops.GA_ERR_UNSUPPORTED
    assert lib.gpt2_attn_decode(None, 5, p, p, p, ws, 2, 1000, 3, 64, 0.125, None) == ops.GA_ERR_INVALID_ARG
    assert lib.gpt2_attn_decode(p, 5, p, p, p, ws, 2, 1000, 3, 64, 0.0, None) == ops.GA_ERR_INVALID_ARG
