"""Python binding of libgpt2attn.so: argument marshalling only.

Every step of the computation runs in the library's CUDA kernels. This module
checks tensor shapes, dtypes and devices, allocates outputs through PyTorch
(which owns device memory and streams), and passes raw pointers and the
current CUDA stream to the C ABI declared in include/gpt2attn.h. If the
library is missing, importing this module raises ImportError: there is no
fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libgpt2attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python -m causal_self_attention_flashattention_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

# Status codes of the C ABI.
GA_OK = 0
GA_ERR_INVALID_ARG = 1
GA_ERR_UNSUPPORTED = 2
GA_ERR_ALIGNMENT = 3
GA_ERR_WORKSPACE = 4
GA_ERR_CUDA = 5
GA_ERR_TIMEOUT = 6
GA_ERR_RANGE = 7

EXPORTED_SYMBOLS = (
    "gpt2_attn_fwd",
    "gpt2_attn_bwd_workspace_size",
    "gpt2_attn_bwd",
    "gpt2_attn_bwd_fused_workspace_size",
    "gpt2_attn_bwd_prepare",
    "gpt2_attn_bwd_fused",
    "gpt2_attn_bwd_preprocess",
    "gpt2_attn_last_cuda_error",
    "gpt2_attn_bwd_dkdv",
    "gpt2_attn_bwd_dq",
    "gpt2_attn_decode_workspace_size",
    "gpt2_attn_decode",
    "gpt2_attn_last_device_status",
    "gpt2_attn_selftest_wait_timeout",
    "gpt2_attn_qkv_proj",
    "gpt2_attn_qkv_proj_v16",
    "gpt2_attn_fwd_v16",
    "gpt2_attn_fp8_quantize",
    "gpt2_attn_fwd_fp8",
    "gpt2_attn_out_proj",
    "gpt2_attn_status_string",
    "gpt2_attn_version",
    "gpt2_attn_fwd_item_schedule",
)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

_lib.gpt2_attn_fwd.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_fwd.restype = _i
_lib.gpt2_attn_bwd_workspace_size.argtypes = [_i, _i, _i, _i, ctypes.POINTER(ctypes.c_size_t)]
_lib.gpt2_attn_bwd_workspace_size.restype = _i
_lib.gpt2_attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                               _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_bwd.restype = _i
_lib.gpt2_attn_bwd_fused_workspace_size.argtypes = [_i, _i, _i, _i,
                                                   ctypes.POINTER(ctypes.c_size_t)]
_lib.gpt2_attn_bwd_fused_workspace_size.restype = _i
_lib.gpt2_attn_bwd_prepare.argtypes = [_vp, _vp, _vp, ctypes.c_size_t, _i, _i, _i, _i, _vp]
_lib.gpt2_attn_bwd_prepare.restype = _i
_lib.gpt2_attn_bwd_fused.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_size_t, _vp,
                                     _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_bwd_fused.restype = _i
_lib.gpt2_attn_last_cuda_error.argtypes = []
_lib.gpt2_attn_last_cuda_error.restype = ctypes.c_ulonglong
_lib.gpt2_attn_bwd_preprocess.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp]
_lib.gpt2_attn_bwd_preprocess.restype = _i
_lib.gpt2_attn_bwd_dkdv.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_bwd_dkdv.restype = _i
_lib.gpt2_attn_bwd_dq.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_bwd_dq.restype = _i
_lib.gpt2_attn_bwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_bwd_noalloc.restype = _i
_lib.gpt2_attn_decode_workspace_size.argtypes = [_i, _i, _i, _i, ctypes.POINTER(ctypes.c_size_t)]
_lib.gpt2_attn_decode_workspace_size.restype = _i
_lib.gpt2_attn_decode.argtypes = [_vp, _i, _vp, _vp, _vp, ctypes.c_size_t, _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_decode.restype = _i
_lib.gpt2_attn_last_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_ulonglong)]
_lib.gpt2_attn_last_device_status.restype = _i
_lib.gpt2_attn_fp8_quantize.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp]
_lib.gpt2_attn_fp8_quantize.restype = _i
_lib.gpt2_attn_fwd_fp8.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_fwd_fp8.restype = _i
_lib.gpt2_attn_qkv_proj.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]
_lib.gpt2_attn_qkv_proj.restype = _i
_lib.gpt2_attn_qkv_proj_v16.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]
_lib.gpt2_attn_qkv_proj_v16.restype = _i
_lib.gpt2_attn_fwd_v16.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]
_lib.gpt2_attn_fwd_v16.restype = _i
_lib.gpt2_attn_out_proj.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]
_lib.gpt2_attn_out_proj.restype = _i
_lib.gpt2_attn_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, _vp]
_lib.gpt2_attn_selftest_wait_timeout.restype = _i
_lib.gpt2_attn_status_string.argtypes = [_i]
_lib.gpt2_attn_status_string.restype = ctypes.c_char_p
_lib.gpt2_attn_version.argtypes = []
_lib.gpt2_attn_version.restype = _i
_ip = ctypes.POINTER(ctypes.c_int)
_lib.gpt2_attn_fwd_item_schedule.argtypes = [_i, _i, _i, _i, _ip, _ip, _ip, ctypes.c_long]
_lib.gpt2_attn_fwd_item_schedule.restype = _i


class AttnError(RuntimeError):
    """A non-zero status from the C ABI."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.gpt2_attn_status_string(int(status)).decode()


def version() -> int:
    return int(_lib.gpt2_attn_version())


def fwd_item_schedule(B: int, T: int, H: int, num_sms: int):
    """The forward's deal of items to launches and CTAs for (B, T, H) on
    num_sms SMs (host code, no GPU needed): int32 arrays (launch, cta, pos)
    indexed by item, and the number of launches. Raises ValueError on bad
    arguments."""
    import numpy as np

    n_items = B * H * (((T + 127) // 128 + 1) // 2) if min(B, T, H) > 0 else 1
    arrs = [np.full(n_items, -1, dtype=np.int32) for _ in range(3)]
    ptrs = [a.ctypes.data_as(_ip) for a in arrs]
    n = _lib.gpt2_attn_fwd_item_schedule(B, T, H, num_sms, *ptrs, n_items)
    if n < 0:
        raise ValueError(f"gpt2_attn_fwd_item_schedule: {status_string(-n)}")
    return arrs[0], arrs[1], arrs[2], n


def _check(status: int, where: str) -> None:
    if status == GA_ERR_CUDA:
        word = int(_lib.gpt2_attn_last_cuda_error())
        step = {1: "device set-up", 2: "TMA descriptor", 3: "kernel launch"}.get(word >> 32, "?")
        raise AttnError(status, f"{where} ({step}: CUDA code {word & 0xFFFFFFFF})")
    if status != GA_OK:
        raise AttnError(status, where)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _expect(t: torch.Tensor, name: str, shape, dtype) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _dims(qkv: torch.Tensor):
    if qkv.dim() != 5 or qkv.shape[2] != 3:
        raise ValueError(f"qkv must be (B, T, 3, H, D), got {tuple(qkv.shape)}")
    B, T, _, H, D = qkv.shape
    return int(B), int(T), int(H), int(D)


def default_scale(D: int) -> float:
    return 1.0 / (D ** 0.5)


def attn_fwd(qkv: torch.Tensor, scale: float | None = None, out: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, stream=None, check_status: bool = False):
    """Causal attention forward: returns (out (B,T,H,D) bf16, lse (B,H,T) fp32).

    The P V product runs in fp16, so every v entry must lie within fp16's
    range (|v| <= 65504, finite). An entry outside it is reported on the
    device as GA_ERR_RANGE, and out is then undefined. The call itself is
    asynchronous and does not see that report; with check_status=True it
    synchronises the stream afterwards and raises AttnError on any device
    report (GA_ERR_RANGE, or GA_ERR_TIMEOUT from a wait that gave up)."""
    B, T, H, D = _dims(qkv)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    scale = default_scale(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=qkv.device)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=qkv.device)
    _expect(out, "out", (B, T, H, D), torch.bfloat16)
    _expect(lse, "lse", (B, H, T), torch.float32)
    _check(_lib.gpt2_attn_fwd(qkv.data_ptr(), out.data_ptr(), lse.data_ptr(), B, T, H, D,
                              scale, _stream_ptr(stream)), "gpt2_attn_fwd")
    if check_status:
        st, word = last_device_status(stream)
        if st != GA_OK:
            raise AttnError(st, f"gpt2_attn_fwd (device report {word:#x})")
    return out, lse


def attn_fwd_v16(qkv: torch.Tensor, scale: float | None = None, out: torch.Tensor | None = None,
                 lse: torch.Tensor | None = None, stream=None):
    """attn_fwd for a qkv whose v slot holds fp16 bits (q, k bf16), as
    qkv_proj(..., v_fp16=True) writes it: returns (out, lse) without the
    kernel's bf16 -> fp16 conversion of V. Inference and prefill only."""
    B, T, H, D = _dims(qkv)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    scale = default_scale(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=qkv.device)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=qkv.device)
    _expect(out, "out", (B, T, H, D), torch.bfloat16)
    _expect(lse, "lse", (B, H, T), torch.float32)
    _check(_lib.gpt2_attn_fwd_v16(qkv.data_ptr(), out.data_ptr(), lse.data_ptr(), B, T, H, D,
                                  scale, _stream_ptr(stream)), "gpt2_attn_fwd_v16")
    return out, lse


def bwd_workspace_size(B: int, T: int, H: int, D: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.gpt2_attn_bwd_workspace_size(B, T, H, D, ctypes.byref(n)),
           "gpt2_attn_bwd_workspace_size")
    return int(n.value)


def attn_bwd(qkv: torch.Tensor, out: torch.Tensor, dout: torch.Tensor, lse: torch.Tensor,
             scale: float | None = None, dqkv: torch.Tensor | None = None,
             workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Causal attention backward: returns dqkv (B,T,3,H,D) bf16 (bitwise deterministic).

    ``workspace`` (a uint8 CUDA tensor of at least ``bwd_workspace_size`` bytes)
    is allocated here when not given; after the call its first B*H*T fp32
    values hold Delta = rowsum(dout * out).
    """
    B, T, H, D = _dims(qkv)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    _expect(out, "out", (B, T, H, D), torch.bfloat16)
    _expect(dout, "dout", (B, T, H, D), torch.bfloat16)
    _expect(lse, "lse", (B, H, T), torch.float32)
    scale = default_scale(D) if scale is None else float(scale)
    if dqkv is None:
        dqkv = torch.empty_like(qkv)
    _expect(dqkv, "dqkv", (B, T, 3, H, D), torch.bfloat16)
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(B, T, H, D), dtype=torch.uint8,
                                device=qkv.device)
    ws, ws_bytes = _workspace(workspace)
    _check(_lib.gpt2_attn_bwd(qkv.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                              dqkv.data_ptr(), ws, ws_bytes, B, T, H, D,
                              scale, _stream_ptr(stream)), "gpt2_attn_bwd")
    return dqkv


def bwd_fused_workspace_size(B: int, T: int, H: int, D: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.gpt2_attn_bwd_fused_workspace_size(B, T, H, D, ctypes.byref(n)),
           "gpt2_attn_bwd_fused_workspace_size")
    return int(n.value)


def _workspace(workspace: torch.Tensor):
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def attn_bwd_fused_steps(qkv: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                         lse: torch.Tensor, workspace: torch.Tensor, dqkv: torch.Tensor,
                         scale: float | None = None, stream=None, events=None) -> torch.Tensor:
    """The fused backward as its two C-ABI steps (prepare, fused kernel).

    ``workspace`` has at least ``bwd_fused_workspace_size`` bytes. Same dqkv as
    ``attn_bwd`` up to fp32 summation order in dq. If ``events`` (three CUDA
    events) is given, they are recorded on the stream before, between and
    after the two launches, so each step can be timed on the device.
    """
    B, T, H, D = _dims(qkv)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    _expect(out, "out", (B, T, H, D), torch.bfloat16)
    _expect(dout, "dout", (B, T, H, D), torch.bfloat16)
    _expect(lse, "lse", (B, H, T), torch.float32)
    _expect(dqkv, "dqkv", (B, T, 3, H, D), torch.bfloat16)
    scale = default_scale(D) if scale is None else float(scale)
    ws, ws_bytes = _workspace(workspace)
    if stream is None:
        stream = torch.cuda.current_stream()
    sp = _stream_ptr(stream)
    if events is not None:
        events[0].record(stream)
    _check(_lib.gpt2_attn_bwd_prepare(out.data_ptr(), dout.data_ptr(), ws, ws_bytes,
                                      B, T, H, D, sp), "gpt2_attn_bwd_prepare")
    if events is not None:
        events[1].record(stream)
    _check(_lib.gpt2_attn_bwd_fused(qkv.data_ptr(), dout.data_ptr(), lse.data_ptr(), ws, ws_bytes,
                                    dqkv.data_ptr(), B, T, H, D, scale, sp), "gpt2_attn_bwd_fused")
    if events is not None:
        events[2].record(stream)
    return dqkv


def attn_bwd_fused(qkv: torch.Tensor, out: torch.Tensor, dout: torch.Tensor, lse: torch.Tensor,
                   scale: float | None = None, dqkv: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The fused backward (gpt2_attn_bwd_prepare + gpt2_attn_bwd_fused)."""
    B, T, H, D = _dims(qkv)
    if dqkv is None:
        dqkv = torch.empty_like(qkv)
    if workspace is None:
        workspace = torch.empty(bwd_fused_workspace_size(B, T, H, D), dtype=torch.uint8,
                                device=qkv.device)
    return attn_bwd_fused_steps(qkv, out, dout, lse, workspace, dqkv, scale, stream)


def attn_bwd_split_steps(qkv: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                         lse: torch.Tensor, delta: torch.Tensor, dqkv: torch.Tensor,
                         scale: float | None = None, stream=None, events=None) -> torch.Tensor:
    """``attn_bwd`` as its two C-ABI steps (dQ, which also writes Delta, then
    dK/dV, which reads it).

    Same result as ``attn_bwd``. ``delta`` is a caller-owned fp32 (B,H,T)
    tensor; on return it holds Delta. If ``events`` (three CUDA events) is
    given, they are recorded on the stream before, between and after the two
    launches, so each step can be timed on the device.
    """
    B, T, H, D = _dims(qkv)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    _expect(out, "out", (B, T, H, D), torch.bfloat16)
    _expect(dout, "dout", (B, T, H, D), torch.bfloat16)
    _expect(lse, "lse", (B, H, T), torch.float32)
    _expect(delta, "delta", (B, H, T), torch.float32)
    _expect(dqkv, "dqkv", (B, T, 3, H, D), torch.bfloat16)
    scale = default_scale(D) if scale is None else float(scale)
    if stream is None:
        stream = torch.cuda.current_stream()
    sp = _stream_ptr(stream)
    if events is not None:
        events[0].record(stream)
    _check(_lib.gpt2_attn_bwd_dq(qkv.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                                 delta.data_ptr(), dqkv.data_ptr(), B, T, H, D, scale, sp),
           "gpt2_attn_bwd_dq")
    if events is not None:
        events[1].record(stream)
    _check(_lib.gpt2_attn_bwd_dkdv(qkv.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                                   delta.data_ptr(), dqkv.data_ptr(), B, T, H, D, scale, sp),
           "gpt2_attn_bwd_dkdv")
    if events is not None:
        events[2].record(stream)
    return dqkv


def attn_bwd_noalloc(qkv: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                     lse: torch.Tensor, scale: float | None = None, dqkv: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """The backward through gpt2_attn_bwd_noalloc: no workspace argument.

    For callers that cannot allocate device memory; Delta lives in the
    library's fixed static scratch (B*H*T <= 2^20), shared by all calls, so
    calls that overlap on the GPU race. Pass a preallocated ``dqkv`` to make
    the call itself allocate nothing.
    """
    B, T, H, D = _dims(qkv)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    _expect(out, "out", (B, T, H, D), torch.bfloat16)
    _expect(dout, "dout", (B, T, H, D), torch.bfloat16)
    _expect(lse, "lse", (B, H, T), torch.float32)
    scale = default_scale(D) if scale is None else float(scale)
    if dqkv is None:
        dqkv = torch.empty_like(qkv)
    _expect(dqkv, "dqkv", (B, T, 3, H, D), torch.bfloat16)
    _check(_lib.gpt2_attn_bwd_noalloc(qkv.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                      lse.data_ptr(), dqkv.data_ptr(), B, T, H, D, scale,
                                      _stream_ptr(stream)), "gpt2_attn_bwd_noalloc")
    return dqkv


def decode_workspace_size(B: int, T: int, H: int, D: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.gpt2_attn_decode_workspace_size(B, T, H, D, ctypes.byref(n)),
           "gpt2_attn_decode_workspace_size")
    return int(n.value)


def attn_decode(qkv: torch.Tensor, t: int, scale: float | None = None,
                out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None):
    """Decode attention of query row ``t`` over rows 0..t of ``qkv``.

    Returns (out (B,H,D) bf16, lse (B,H) fp32): row t of ``attn_fwd``'s result.
    """
    B, T, H, D = _dims(qkv)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    scale = default_scale(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.bfloat16, device=qkv.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=qkv.device)
    _expect(out, "out", (B, H, D), torch.bfloat16)
    _expect(lse, "lse", (B, H), torch.float32)
    if workspace is None:
        workspace = torch.empty(decode_workspace_size(B, T, H, D), dtype=torch.uint8,
                                device=qkv.device)
    ws, ws_bytes = _workspace(workspace)
    _check(_lib.gpt2_attn_decode(qkv.data_ptr(), int(t), out.data_ptr(), lse.data_ptr(), ws,
                                 ws_bytes, B, T, H, D, scale, _stream_ptr(stream)),
           "gpt2_attn_decode")
    return out, lse


def last_device_status(stream=None) -> tuple[int, int]:
    """Synchronises the stream; returns (status, raw status word) and clears it."""
    word = ctypes.c_ulonglong(0)
    st = _lib.gpt2_attn_last_device_status(_stream_ptr(stream), ctypes.byref(word))
    return int(st), int(word.value)


class CausalSelfAttention(torch.autograd.Function):
    """Autograd wrapper: y = attention(qkv), with both passes in the library.
    The forward's fp16 limit on v applies (see attn_fwd)."""

    @staticmethod
    def forward(ctx, qkv, scale=None, check_status=False):
        out, lse = attn_fwd(qkv, scale, check_status=check_status)
        ctx.save_for_backward(qkv, out, lse)
        ctx.scale = scale
        return out

    @staticmethod
    def backward(ctx, dout):
        qkv, out, lse = ctx.saved_tensors
        return attn_bwd(qkv, out, dout.contiguous(), lse, ctx.scale), None, None


def causal_self_attention(qkv: torch.Tensor, scale: float | None = None,
                          check_status: bool = False) -> torch.Tensor:
    """One-call causal self-attention on packed qkv (B,T,3,H,D) -> (B,T,H,D).

    Every v entry must lie within fp16's range (|v| <= 65504): the forward's
    P V product runs in fp16. check_status=True synchronises after the
    forward and raises AttnError if the device reported a v entry outside it
    (or a wait that gave up); otherwise out is undefined in that case."""
    return CausalSelfAttention.apply(qkv, scale, check_status)


def qkv_proj(x: torch.Tensor, w_attn: torch.Tensor, b_attn: torch.Tensor, H: int,
             qkv: torch.Tensor | None = None, stream=None, v_fp16: bool = False) -> torch.Tensor:
    """c_attn: qkv = x W_attn^T + b_attn, returned as packed (B, T, 3, H, D) bf16.

    x (B, T, C) bf16, w_attn (3C, C) bf16 (nn.Linear layout), b_attn (3C,) bf16.
    With v_fp16=True the v slot holds fp16 bits (read it as
    qkv[:, :, 2].view(torch.float16)): the input of attn_fwd_v16, not of
    attn_fwd or attn_bwd.
    """
    if x.dim() != 3:
        raise ValueError(f"x must be (B, T, C), got {tuple(x.shape)}")
    B, T, C = (int(d) for d in x.shape)
    if C % H:
        raise ValueError("C must be a multiple of H")
    D = C // H
    _expect(x, "x", (B, T, C), torch.bfloat16)
    _expect(w_attn, "w_attn", (3 * C, C), torch.bfloat16)
    _expect(b_attn, "b_attn", (3 * C,), torch.bfloat16)
    if qkv is None:
        qkv = torch.empty((B, T, 3, H, D), dtype=torch.bfloat16, device=x.device)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    fn = _lib.gpt2_attn_qkv_proj_v16 if v_fp16 else _lib.gpt2_attn_qkv_proj
    _check(fn(x.data_ptr(), w_attn.data_ptr(), b_attn.data_ptr(), qkv.data_ptr(), B, T, H, D,
              _stream_ptr(stream)),
           "gpt2_attn_qkv_proj_v16" if v_fp16 else "gpt2_attn_qkv_proj")
    return qkv


def out_proj(out: torch.Tensor, w_proj: torch.Tensor, b_proj: torch.Tensor,
             y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """c_proj: y = out W_proj^T + b_proj from the attention output (B, T, H, D);
    returns y (B, T, C) bf16. w_proj (C, C) bf16, b_proj (C,) bf16."""
    if out.dim() != 4:
        raise ValueError(f"out must be (B, T, H, D), got {tuple(out.shape)}")
    B, T, H, D = (int(d) for d in out.shape)
    C = H * D
    _expect(out, "out", (B, T, H, D), torch.bfloat16)
    _expect(w_proj, "w_proj", (C, C), torch.bfloat16)
    _expect(b_proj, "b_proj", (C,), torch.bfloat16)
    if y is None:
        y = torch.empty((B, T, C), dtype=torch.bfloat16, device=out.device)
    _expect(y, "y", (B, T, C), torch.bfloat16)
    _check(_lib.gpt2_attn_out_proj(out.data_ptr(), w_proj.data_ptr(), b_proj.data_ptr(),
                                   y.data_ptr(), B, T, H, D, _stream_ptr(stream)),
           "gpt2_attn_out_proj")
    return y


def fp8_quantize(qkv: torch.Tensor, qkv8: torch.Tensor | None = None,
                 scales: torch.Tensor | None = None, stream=None):
    """Per-tensor e4m3 quantisation of q, k, v: returns (qkv8 (B,T,3,H,D)
    uint8 e4m3 bytes, scales fp32[8] whose [0..2] are the dequantisation
    multipliers)."""
    B, T, H, D = _dims(qkv)
    _expect(qkv, "qkv", (B, T, 3, H, D), torch.bfloat16)
    if qkv8 is None:
        qkv8 = torch.empty((B, T, 3, H, D), dtype=torch.uint8, device=qkv.device)
    if scales is None:
        scales = torch.empty(8, dtype=torch.float32, device=qkv.device)
    _expect(qkv8, "qkv8", (B, T, 3, H, D), torch.uint8)
    _expect(scales, "scales", (8,), torch.float32)
    _check(_lib.gpt2_attn_fp8_quantize(qkv.data_ptr(), qkv8.data_ptr(), scales.data_ptr(),
                                       B, T, H, D, _stream_ptr(stream)), "gpt2_attn_fp8_quantize")
    return qkv8, scales


def attn_fwd_fp8(qkv8: torch.Tensor, scales: torch.Tensor, scale: float | None = None,
                 out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """FP8 forward from fp8_quantize's output: returns (out bf16, lse fp32)."""
    B, T, H, D = _dims(qkv8)
    _expect(qkv8, "qkv8", (B, T, 3, H, D), torch.uint8)
    _expect(scales, "scales", (8,), torch.float32)
    scale = default_scale(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=qkv8.device)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=qkv8.device)
    _expect(out, "out", (B, T, H, D), torch.bfloat16)
    _expect(lse, "lse", (B, H, T), torch.float32)
    _check(_lib.gpt2_attn_fwd_fp8(qkv8.data_ptr(), scales.data_ptr(), out.data_ptr(),
                                  lse.data_ptr(), B, T, H, D, scale, _stream_ptr(stream)),
           "gpt2_attn_fwd_fp8")
    return out, lse
