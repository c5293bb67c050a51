"""NVFP4 weight decoding from the format's definition (test infrastructure; see oracle/__init__).

The pages give NVFP4 as the weight format behind their lowest bytes-per-token
roofline ("Ultra-High Interactivity On NVIDIA GPUs? - TileRT InferenceX",
digest, core views: ~21 GB of active parameters per token for GLM-5 in NVFP4).
The format: each element is an E2M1 code (1 sign bit, 2 exponent bits with
bias 1, 1 mantissa bit, a subnormal when the exponent field is 0, no
infinities or NaN; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6); every 16
consecutive elements of a row share one E4M3 scale, and the tensor has one
fp32 scale.  An element's value is code * block scale * tensor scale.

Storage (as the C ABI takes it): codes uint8 [N][K/2], element 2j in the low
nibble of byte j and element 2j+1 in the high nibble; block scales uint8
e4m3 codes [N][K/16]; the tensor scale one fp32 value.
"""
from __future__ import annotations

import math

import torch

from .fp8 import e4m3_to_fp32


def _decode_one(code: int) -> float:
    sign = -1.0 if code & 0x8 else 1.0
    exp_field = (code >> 1) & 0x3
    mant = code & 0x1
    if exp_field == 0:
        return sign * math.ldexp(mant / 2.0, 1 - 1)
    return sign * math.ldexp(1.0 + mant / 2.0, exp_field - 1)


def e2m1_decode_table() -> torch.Tensor:
    """fp32 value of each of the 16 codes."""
    return torch.tensor([_decode_one(c) for c in range(16)], dtype=torch.float32)


def nvfp4_dequant(codes: torch.Tensor, scales: torch.Tensor, tensor_scale: float) -> torch.Tensor:
    """fp32 [N][K] values of an NVFP4 matrix: code * e4m3 block scale * tensor scale."""
    N, half = codes.shape
    K = 2 * half
    assert scales.shape == (N, K // 16), (scales.shape, N, K)
    table = e2m1_decode_table()
    c = codes.long()
    vals = torch.stack([table[c & 0xF], table[c >> 4]], dim=-1).view(N, K)   # even, odd elements
    block = e4m3_to_fp32(scales).repeat_interleave(16, dim=1)                 # [N][K]
    return vals * block * float(tensor_scale)
