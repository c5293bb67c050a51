"""FP8 e4m3 decoding and encoding from the format's definition (test infrastructure; see oracle/__init__).

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


def e4m3_encode(x: torch.Tensor) -> torch.Tensor:
    """uint8 e4m3 codes of fp32 values: round to the nearest representable
    value, ties to the even code (mantissa LSB 0), magnitudes beyond the largest
    finite value saturate to +-448 (the "satfinite" conversion).  Written from
    the format: the non-negative finite codes 0x00..0x7E are increasing in value,
    so the nearest one is found by a search over their value table."""
    global _TABLE
    if _TABLE is None:
        _TABLE = e4m3_decode_table()
    pos = _TABLE[:0x7F]                                   # values of codes 0x00..0x7E, increasing
    xf = x.float().reshape(-1)
    a = xf.abs().clamp(max=448.0)
    hi = torch.searchsorted(pos, a).clamp(max=0x7E)       # first code with value >= a
    lo = (hi - 1).clamp(min=0)
    d_hi = pos[hi] - a
    d_lo = a - pos[lo]
    take_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0) & (lo != hi))
    code = torch.where(take_lo, lo, hi)
    sign = (xf < 0) | ((xf == 0) & torch.signbit(xf))
    code = code | (sign.to(torch.int64) << 7)
    return code.to(torch.uint8).reshape(x.shape)
