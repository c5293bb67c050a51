"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This package holds model shapes and counter-based random generators only: it
contains none of the decoder's arithmetic (no norm, projection, attention,
activation or routing).  Both sides of every parity test draw their inputs from
here, on the host or on a CUDA device, bit-identically.
"""
from .configs import DecoderConfig, CONFIGS, fp8_kv, get_config  # noqa: F401
from .gen import (  # noqa: F401
    splitmix64_stream,
    normal_bf16,
    normal_fp32,
    uniform_tokens,
    quantize_fp8_blocks,
    quantize_nvfp4,
    make_weights,
    make_prompt,
    make_synthetic_kv,
    fp8_kv_values,
    fp8_kv_codes,
    make_start_tokens,
    stream_key,
)
