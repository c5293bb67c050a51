"""FP8 e4m3 decoding from the format's definition (test infrastructure; see oracle/__init__).

The FP8 weights of the block-scaled workload are e4m3 codes (TileRT ships FP8
weights in production: "Ultra-High Interactivity On NVIDIA GPUs? - TileRT
InferenceX", digest, InferenceX results; "TileRT speed notes", FP8 section).
The format is the OCP 8-bit "E4M3" encoding: 1 sign bit, 4 exponent bits with
bias 7, 3 mantissa bits, subnormals when the exponent field is 0, no
infinities, and the two codes S.1111.111 are NaN; the largest finite
magnitude is 1.75 * 2^8 = 448.
"""
from __future__ import annotations

import math

import torch


def _decode_one(code: int) -> float:
    sign = -1.0 if code & 0x80 else 1.0
    exp_field = (code >> 3) & 0xF
    mant = code & 0x7
    if exp_field == 0xF and mant == 0x7:
        return math.nan
    if exp_field == 0:
        return sign * math.ldexp(mant / 8.0, 1 - 7)
    return sign * math.ldexp(1.0 + mant / 8.0, exp_field - 7)


def e4m3_decode_table() -> torch.Tensor:
    """fp32 value of each of the 256 codes (exact: every e4m3 value is an fp32 value)."""
    return torch.tensor([_decode_one(c) for c in range(256)], dtype=torch.float32)


_TABLE = None


def e4m3_to_fp32(codes: torch.Tensor) -> torch.Tensor:
    """Widen uint8 e4m3 codes to fp32 by table lookup."""
    global _TABLE
    if _TABLE is None:
        _TABLE = e4m3_decode_table()
    return _TABLE[codes.long()]
