"""Decoder shapes of the synthetic workloads.

The workloads are the Llama-style decoders named for this hot path (a tiny
2-layer model, a 1B shape, an 8B shape in bf16 and in block-scaled FP8, and a
top-8 MoE shape).  The pages measure TileRT on InferenceX with GLM-5.1 ("Ultra-
High Interactivity On NVIDIA GPUs? - TileRT InferenceX", digest, InferenceX
results); neither that suite nor any trained weight is available, so these
seeded random-init models stand in for it.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class DecoderConfig:
    name: str
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int              # dense SwiGLU width (0 for MoE layers)
    vocab: int
    kv_len: int           # positions already in the KV cache when timed decode starts
    steps: int            # greedy decode steps of one workload pass
    batch: int = 1
    weight_dtype: str = "bf16"   # "bf16" or "fp8_e4m3" (fp32 scale per 128x128 block)
    n_experts: int = 0
    top_k: int = 0
    n_shared_experts: int = 0
    expert_ffn: int = 0
    rope_theta: float = 1.0e4
    rms_eps: float = 1.0e-5
    init_std: float = 0.02
    prefill: bool = True   # KV from a seeded prompt (True) or seeded synthetic KV (False)
    seed: int = 0
    kv_dtype: str = "bf16"   # "bf16" or "fp8_e4m3" (one power-of-two scale per tensor)
    k_scale: float = 0.0     # e4m3 cache: scales of K and V entries (powers of two)
    v_scale: float = 0.0

    @property
    def max_seq(self) -> int:
        return self.kv_len + self.steps

    @property
    def is_moe(self) -> bool:
        return self.n_experts > 0

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def with_(self, **kw) -> "DecoderConfig":
        return dataclasses.replace(self, **kw)

    def weight_bytes_per_elem(self) -> float:
        return {"fp8_e4m3": 1, "nvfp4": 0.5}.get(self.weight_dtype, 2)


TINY = DecoderConfig(
    name="tiny", n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
    ffn=1024, vocab=4096, kv_len=128, steps=32)

LLAMA_1B = DecoderConfig(
    name="llama1b", n_layers=16, hidden=2048, n_q_heads=32, n_kv_heads=8, head_dim=64,
    ffn=8192, vocab=32000, kv_len=1024, steps=256)

LLAMA_8B = DecoderConfig(
    name="llama8b", n_layers=32, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
    ffn=14336, vocab=128256, kv_len=8192, steps=256, prefill=False)

LLAMA_8B_FP8 = LLAMA_8B.with_(name="llama8b_fp8", weight_dtype="fp8_e4m3", kv_len=1024)

LLAMA_8B_NVFP4 = LLAMA_8B.with_(name="llama8b_nvfp4", weight_dtype="nvfp4")

MOE = DecoderConfig(
    name="moe", n_layers=24, hidden=2048, n_q_heads=16, n_kv_heads=4, head_dim=128,
    ffn=0, vocab=64000, kv_len=4096, steps=256, n_experts=64, top_k=8,
    n_shared_experts=1, expert_ffn=1408, prefill=False)

CONFIGS = {c.name: c for c in (TINY, LLAMA_1B, LLAMA_8B, LLAMA_8B_FP8, LLAMA_8B_NVFP4, MOE)}


def fp8_kv(cfg: DecoderConfig) -> DecoderConfig:
    """The same model with an e4m3 KV cache.  K and V entries are about
    N(0, (init_std * sqrt(hidden))^2) (a projection of a unit-RMS activation); the
    scale is the power of two that puts 6 sigma just under e4m3's largest value 448."""
    import math
    sigma = cfg.init_std * math.sqrt(cfg.hidden)
    scale = 2.0 ** math.ceil(math.log2(6.0 * sigma / 448.0))
    return cfg.with_(kv_dtype="fp8_e4m3", k_scale=scale, v_scale=scale)


def get_config(name: str, **overrides) -> DecoderConfig:
    cfg = CONFIGS[name]
    return cfg.with_(**overrides) if overrides else cfg
