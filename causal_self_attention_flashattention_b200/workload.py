"""Seeded synthetic inputs for causal self-attention at GPT-2 shapes.

This module only draws random numbers. It holds none of the attention
arithmetic, and both the CUDA path and the CPU oracle take their inputs from
it.

The pages train GPT-2 (124M: 12 layers, width 768, 12 heads of 64) on
FineWeb-Edu ("Let's reproduce GPT-2 (124M)" video summary page, closing
summary paragraph). That dataset and the trained weights are not available
here, and attention needs only its activations. So seeded Gaussians stand in
for the packed ``c_attn`` output (B, T, 3, H, D) and for the upstream gradient
dO (B, T, H, D):

* a CPU ``torch.Generator`` seeded with ``seed``;
* qkv = randn(B, T, 3, H, D) in fp32, then dO = randn(B, T, H, D) from the
  same generator;
* the q and k slots are multiplied by ``qk_std`` (3.0 for the long-context
  stress case, which gives peaked softmax rows); this happens before rounding;
* both are rounded to bf16 (round-to-nearest-even), which is what both sides
  see.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_linear_inputs", "attention_flops",
           "algorithmic_bytes"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    D: int = 64
    qk_std: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / (self.D ** 0.5)


# The five attention shapes of the GPT-2 reproduction (124M and 350M model
# widths, micro-batch 16 and 64, plus a 4096-token stress case).
WORKLOADS = {
    "gpt2-124m-b1-t128": Workload("gpt2-124m-b1-t128", 1, 128, 12),
    "gpt2-124m-b16-t1024": Workload("gpt2-124m-b16-t1024", 16, 1024, 12),
    "gpt2-124m-b64-t1024": Workload("gpt2-124m-b64-t1024", 64, 1024, 12),
    "gpt2-350m-b32-t1024": Workload("gpt2-350m-b32-t1024", 32, 1024, 16),
    "stress-b4-t4096-qk3": Workload("stress-b4-t4096-qk3", 4, 4096, 12, qk_std=3.0),
    # A quarter of the bench batch: the size the full ncu captures run at.
    "gpt2-124m-b4-t1024": Workload("gpt2-124m-b4-t1024", 4, 1024, 12),
}


def make_inputs(B: int, T: int, H: int, D: int = 64, seed: int = 0, qk_std: float = 1.0):
    """Returns (qkv, dout) as CPU bf16 tensors, shapes (B,T,3,H,D) and (B,T,H,D)."""
    g = torch.Generator().manual_seed(int(seed))
    qkv = torch.randn(B, T, 3, H, D, dtype=torch.float32, generator=g)
    dout = torch.randn(B, T, H, D, dtype=torch.float32, generator=g)
    if qk_std != 1.0:
        qkv[:, :, 0:2] *= qk_std
    return qkv.to(torch.bfloat16), dout.to(torch.bfloat16)


def make_linear_inputs(B: int, T: int, C: int, n_out: int, seed: int = 0):
    """Returns (x, w, b) for a dense layer C -> n_out as CPU bf16 tensors:
    x (B, T, C) ~ N(0, 1) (the normalised activations a GPT-2 block feeds its
    layers), w (n_out, C) and b (n_out,) ~ N(0, 0.02^2) (GPT-2's weight
    initialisation scale; the bias is drawn too so that its addition is
    exercised)."""
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(B, T, C, dtype=torch.float32, generator=g)
    w = torch.randn(n_out, C, dtype=torch.float32, generator=g) * 0.02
    b = torch.randn(n_out, dtype=torch.float32, generator=g) * 0.02
    return x.to(torch.bfloat16), w.to(torch.bfloat16), b.to(torch.bfloat16)


def attention_flops(B: int, T: int, H: int, D: int) -> tuple[float, float]:
    """Nominal causal FLOPs (forward, backward): 2*B*H*T^2*D and 2.5x that."""
    fwd = 2.0 * B * H * T * T * D
    return fwd, 2.5 * fwd


def algorithmic_bytes(B: int, T: int, H: int, D: int) -> tuple[int, int]:
    """Minimum HBM bytes (forward, backward) the method must move.

    forward : read qkv (bf16), write out (bf16) and lse (fp32)
    backward: read qkv, out, dout, lse; write dqkv; write and read Delta (fp32)
    """
    qkv = B * T * 3 * H * D * 2
    o = B * T * H * D * 2
    lse = B * H * T * 4
    fwd = qkv + o + lse
    bwd = qkv + o + o + lse + qkv + 2 * lse
    return fwd, bwd
