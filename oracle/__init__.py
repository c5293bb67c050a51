"""Oracle: a plain, slow, obviously correct CPU decoder forward (test infrastructure).

This package is test infrastructure.  Only the test suite, the smoke check and
the bench's CPU-baseline / reference arm may import it; the library's product
path never calls it and has no CPU fallback.  It shares no code with the CUDA
path: the two meet only in the seeded input generators of `synth`.

Precision: fp32 throughout (a plain fp32 CPU decode forward), with the KV cache
held exactly like the device cache: bf16 entries, or e4m3 codes times one
power-of-two scale per tensor.  Weights keep their stored bytes (bf16; e4m3
codes with fp32 128x128 block scales; or NVFP4 e2m1 codes with an e4m3 scale
per 16 columns and an fp32 matrix scale) and are widened to fp32 on use.

Parity pins: every function here is pinned by a `-m "not gpu"` test to
something other than itself (library routines, closed forms, invariants,
brute force); see tests/test_oracle_pins.py.  The end-to-end decode of the
synthetic models has no printed worked example on the pages: beyond those pins
it is "parity unpinned" (no page prints a decoded sequence or logit for them).
"""
from .fp8 import e4m3_decode_table, e4m3_encode, e4m3_to_fp32  # noqa: F401
from .fp4 import e2m1_decode_table, nvfp4_dequant  # noqa: F401
from .decoder import (  # noqa: F401
    rms_norm,
    rope_rotate,
    rope_angles,
    attention_decode,
    silu,
    swiglu_ffn,
    moe_route,
    argmax_lowest,
    OracleDecoder,
)
