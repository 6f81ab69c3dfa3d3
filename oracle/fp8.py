"""Per-tensor e4m3 quantisation of q, k and v, as an FP8 forward reads them.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only the test suite may. It shares no code with the CUDA library.

The llm.c page says training runs in BF16 and that FP8 support is planned
("Réimplémenter à bas coût le modèle GPT-2 avec llm.c", FAQ entry on FP8
training). The pages fix no FP8 format or scaling, so the plainest reading is
taken: one scale per tensor (q, k and v of the packed (B, T, 3, H, D) buffer
each get their own), chosen so that the tensor's largest magnitude lands on
the largest e4m3 value, 448:

    amax_s = max |x| over slot s            (0 -> scale 1)
    scale_s = fp32(448 / amax_s)            (the quantising multiplier)
    x8 = e4m3(fp32(x * scale_s))            (round to nearest even)
    dequant_s = fp32(amax_s / 448)          (the multiplier back)

and the dequantised input the attention sees is x8 * dequant_s. All fp32
steps are single correctly rounded operations. An FP8 forward is then checked
against the fp64 oracle on these dequantised inputs (the attention it
computes), not on the bf16 inputs (the attention it was asked for): the e4m3
rounding of the inputs alone moves the result far beyond the bf16 path's
tolerances.

The e4m3 rounding itself is torch's float8_e4m3fn conversion (a library
primitive: round to nearest even; finite values up to 448).
"""

from __future__ import annotations

import numpy as np
import torch

E4M3_MAX = 448.0


def slot_amax(qkv):
    """max |x| of each slot s of qkv (B, T, 3, H, D): float32 (3,)."""
    x = np.abs(np.asarray(qkv, dtype=np.float32))
    return np.array([x[:, :, s].max() if x[:, :, s].size else 0.0 for s in range(3)],
                    dtype=np.float32)


def scales(amax):
    """(scale, dequant) per slot: fp32(448 / amax), fp32(amax / 448); 1, 1 for amax 0."""
    amax = np.asarray(amax, dtype=np.float32)
    q = np.where(amax > 0, np.float32(E4M3_MAX) / np.where(amax > 0, amax, 1), 1)
    d = np.where(amax > 0, amax / np.float32(E4M3_MAX), 1)
    return q.astype(np.float32), d.astype(np.float32)


def e4m3_bits(x):
    """Round float32 values to e4m3 (nearest even): the byte patterns, uint8."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_value(bits):
    """The float32 values of e4m3 byte patterns."""
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float32).numpy()


def quantize_qkv(qkv):
    """qkv (B, T, 3, H, D) -> (bytes uint8 of the same shape, dequant (3,) fp32)."""
    x = np.asarray(qkv, dtype=np.float32)
    q, d = scales(slot_amax(x))
    scaled = (x * q[None, None, :, None, None]).astype(np.float32)
    return e4m3_bits(scaled), d


def dequantize_qkv(bits, dequant):
    """The fp64 inputs an FP8 forward computes with: e4m3 value * dequant."""
    v = e4m3_value(bits).astype(np.float64)
    return v * np.asarray(dequant, dtype=np.float64)[None, None, :, None, None]
