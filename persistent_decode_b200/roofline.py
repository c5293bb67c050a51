"""Algorithmic bytes of one decode step and the bandwidth roofline.

The pages bound decode speed by memory bandwidth: tokens per second per user
cannot exceed HBM bandwidth divided by the bytes each token must read
("Ultra-High Interactivity On NVIDIA GPUs? - TileRT InferenceX", digest, the
bandwidth-roofline paragraph: 64 TB/s over ~21 GB of active parameters gives
3,047 tok/s/user; "TileRT speed notes": ~38 TB/s over ~42 GB gives ~1000
tok/s).  Here the bytes of one step are the weights actually streamed (all
linear layers including the LM head, the norm gains and one embedding row per
sequence) plus, per sequence, the KV cache read at the step's length and the
new K/V entries written.
"""
from __future__ import annotations


def weight_bytes(cfg) -> int:
    if cfg.weight_dtype == "nvfp4":
        return _nvfp4_weight_bytes(cfg)
    esz = 1 if cfg.weight_dtype == "fp8_e4m3" else 2
    H, qd, kvd = cfg.hidden, cfg.q_dim, cfg.kv_dim
    per_layer = (qd + 2 * kvd) * H + H * qd
    if cfg.is_moe:
        Fe = cfg.expert_ffn
        per_layer += (cfg.top_k + cfg.n_shared_experts) * 3 * Fe * H
        router = cfg.n_experts * H * 2
    else:
        per_layer += 3 * cfg.ffn * H
        router = 0
    lin = (cfg.n_layers * per_layer + cfg.vocab * H) * esz
    scales = 0
    if esz == 1:
        scales = 4 * (cfg.n_layers * per_layer + cfg.vocab * H) // (128 * 128)
    norms = 4 * H * (2 * cfg.n_layers + 1)
    return lin + scales + norms + cfg.n_layers * router


def _nvfp4_weight_bytes(cfg) -> int:
    """NVFP4 (dense): half a byte per element, one e4m3 scale byte per 16
    elements, one fp32 scale per matrix; norm gains fp32."""
    H, qd, kvd = cfg.hidden, cfg.q_dim, cfg.kv_dim
    mats = [qd * H, kvd * H, kvd * H, H * qd, cfg.ffn * H, cfg.ffn * H, H * cfg.ffn]
    elems = cfg.n_layers * sum(mats) + cfg.vocab * H
    n_mats = cfg.n_layers * len(mats) + 1
    norms = 4 * H * (2 * cfg.n_layers + 1)
    return elems // 2 + elems // 16 + 4 * n_mats + norms


def step_bytes(cfg, kv_positions: int, batch: int = None) -> int:
    """Bytes of one decode step whose new token lands at position `kv_positions`
    (so kv_positions + 1 entries are attended per sequence)."""
    B = cfg.batch if batch is None else batch
    kv_esz = 1 if getattr(cfg, "kv_dtype", "bf16") == "fp8_e4m3" else 2
    kv_entry = cfg.n_layers * cfg.n_kv_heads * cfg.head_dim * 2 * kv_esz   # K and V entries
    per_seq = kv_entry * (kv_positions + 1) + kv_entry + cfg.hidden * 2  # read, write, embed row
    return weight_bytes(cfg) + B * per_seq


def call_bytes(cfg, start: int, n_steps: int, batch: int = None) -> int:
    """Bytes of n_steps consecutive steps starting with `start` cached positions."""
    return sum(step_bytes(cfg, start + s, batch) for s in range(n_steps))


def tok_per_s_bound(bytes_per_token: float, bandwidth_bytes_per_s: float) -> float:
    return bandwidth_bytes_per_s / bytes_per_token
