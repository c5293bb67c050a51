"""Construction of the seeded synthetic decode workloads on a CUDA device.

Shared by the tests and bench.py: weights and KV contents come from the
seeded generators in `synth` (generated directly on the device), the engine
is created through the C ABI, and the prompt state is set up either by a
teacher-forced prefill through the engine (prompt workloads) or by writing the
seeded synthetic cache (synthetic-KV workloads).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

import synth
from .engine import Engine


@dataclasses.dataclass
class GpuModel:
    cfg: object
    weights: Dict[str, torch.Tensor]
    k: torch.Tensor
    v: torch.Tensor
    engine: Engine
    prompt: Optional[torch.Tensor]      # [B][kv_len+1] for prompt workloads
    start_tokens: torch.Tensor           # [B] pending token when decode starts (host int32)


def kv_shape(cfg, batch: int, max_seq: int):
    return (cfg.n_layers, batch, cfg.n_kv_heads, max_seq, cfg.head_dim)


def build(cfg, device="cuda", norm_std: float = 0.0, n_ctas: int = 0, max_seq: Optional[int] = None,
          spin_limit_us: int = 0, weights: Optional[Dict[str, torch.Tensor]] = None, flags: int = 0,
          window: int = 0) -> GpuModel:
    dev = torch.device(device)
    B = cfg.batch
    ms = max_seq if max_seq is not None else cfg.max_seq
    w = weights if weights is not None else synth.make_weights(cfg, device=dev, norm_std=norm_std)
    k = torch.zeros(kv_shape(cfg, B, ms), dtype=torch.bfloat16, device=dev)
    v = torch.zeros_like(k)
    prompt = None
    if cfg.prefill:
        prompt = synth.make_prompt(cfg, device="cpu")
        start = prompt[:, cfg.kv_len].clone()
    else:
        for l in range(cfg.n_layers):
            kl, vl = synth.make_synthetic_kv(cfg, l, device=dev)
            k[l, :, :, : cfg.kv_len] = kl
            v[l, :, :, : cfg.kv_len] = vl
        start = synth.make_start_tokens(cfg, device="cpu")
    eng = Engine(cfg, w, k, v, n_ctas=n_ctas, spin_limit_us=spin_limit_us, flags=flags, window=window)
    m = GpuModel(cfg, w, k, v, eng, prompt, start.to(torch.int32))
    if cfg.prefill:
        prefill(m)
    return m


def prefill(m: GpuModel, unfused: bool = False) -> None:
    """Teacher-forced prefill of the prompt through the engine: afterwards the cache
    holds kv_len positions and the pending token is prompt[:, kv_len]."""
    cfg = m.cfg
    T = cfg.kv_len
    dev = m.k.device
    m.engine.set_state(m.prompt[:, 0].tolist(), [0] * cfg.batch)
    if T > 0:
        forced = m.prompt[:, 1:T + 1].t().contiguous().to(dev)          # [T][B]
        out = torch.empty(T, cfg.batch, dtype=torch.int32, device=dev)
        m.engine.decode(T, out, forced=forced, unfused=unfused)
    m.engine.check()


def reset_state(m: GpuModel) -> None:
    """Back to the start of timed decode (positions >= kv_len are rewritten before use)."""
    m.engine.set_state(m.start_tokens.tolist(), [m.cfg.kv_len] * m.cfg.batch)
