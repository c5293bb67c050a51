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
    k: torch.Tensor                      # [L][B][n_kv][max_seq][d], or paged: [L][n_pages][n_kv][P][d]
    v: torch.Tensor
    engine: Engine
    prompt: Optional[torch.Tensor]      # [B][kv_len+1] for prompt workloads
    start_tokens: torch.Tensor           # [B] pending token when decode starts (host int32)
    page_table: Optional[torch.Tensor] = None   # paged cache: int32 [B][pages per sequence]


def kv_shape(cfg, batch: int, max_seq: int):
    return (cfg.n_layers, batch, cfg.n_kv_heads, max_seq, cfg.head_dim)


def page_size(cfg) -> int:
    """Positions per page of a paged cache: one attention chunk (32 KB of K and V)."""
    return 16384 // (cfg.head_dim * 2)


def make_page_table(B: int, pages_per_seq: int, n_pages: int, seed: int = 7,
                    shared_prefix_pages: int = 0) -> torch.Tensor:
    """A seeded scattered page table int32 [B][pages_per_seq]: the pool's pages in a
    random order (sequence b takes the next pages_per_seq of the permutation).  With
    shared_prefix_pages, every sequence's first pages are sequence 0's."""
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g).to(torch.int32)
    t = perm[: B * pages_per_seq].view(B, pages_per_seq).clone()
    if shared_prefix_pages:
        t[:, :shared_prefix_pages] = t[0, :shared_prefix_pages]
    return t


def contiguous_view(m: "GpuModel", which: str = "k") -> torch.Tensor:
    """The cache as [L][B][n_kv][max_seq][d], gathered from the pages of a paged cache."""
    c = getattr(m, which)
    if m.page_table is None:
        return c
    pt = m.page_table.to(c.device).long()                       # [B][np]
    g = c[:, pt]                                                 # [L][B][np][n_kv][P][d]
    L, B, npg, nkv, P, d = g.shape
    return g.permute(0, 1, 3, 2, 4, 5).reshape(L, B, nkv, npg * P, d)[:, :, :, : m.engine.max_seq]


def kv_dtype(cfg) -> torch.dtype:
    """Element type of the cache tensors: bf16, or uint8 e4m3 codes."""
    return torch.uint8 if getattr(cfg, "kv_dtype", "bf16") == "fp8_e4m3" else torch.bfloat16


def kv_values(m: "GpuModel", which: str = "k") -> torch.Tensor:
    """The cache entries' values as bf16 [L][B][n_kv][max_seq][d] (an e4m3 cache:
    code * scale, exact in bf16)."""
    c = contiguous_view(m, which)
    if c.dtype != torch.uint8:
        return c
    scale = m.cfg.k_scale if which == "k" else m.cfg.v_scale
    return (c.view(torch.float8_e4m3fn).float() * scale).to(torch.bfloat16)


def build(cfg, device="cuda", norm_std: float = 0.0, n_ctas: int = 0, max_seq: Optional[int] = None,
          spin_limit_us: int = 0, weights: Optional[Dict[str, torch.Tensor]] = None, flags: int = 0,
          window: int = 0, paged: bool = False, spare_pages: int = 3, shared_prefix_pages: int = 0,
          page_seed: int = 7, same_prompt: bool = False) -> GpuModel:
    """A seeded workload on the device with its engine.  `paged` puts the cache in a
    scattered page pool (make_page_table) with `spare_pages` pages nobody uses;
    `same_prompt` gives every sequence sequence 0's prompt (shared-prefix tests)."""
    dev = torch.device(device)
    B = cfg.batch
    ms = max_seq if max_seq is not None else cfg.max_seq
    w = weights if weights is not None else synth.make_weights(cfg, device=dev, norm_std=norm_std)
    pt = None
    if paged:
        P = page_size(cfg)
        nps = (ms + P - 1) // P
        n_pages = B * nps + spare_pages
        pt = make_page_table(B, nps, n_pages, page_seed, shared_prefix_pages)
        k = torch.zeros((cfg.n_layers, n_pages, cfg.n_kv_heads, P, cfg.head_dim), dtype=kv_dtype(cfg),
                        device=dev)
    else:
        k = torch.zeros(kv_shape(cfg, B, ms), dtype=kv_dtype(cfg), device=dev)
    v = torch.zeros_like(k)
    prompt = None
    if cfg.prefill:
        prompt = synth.make_prompt(cfg, device="cpu")
        if same_prompt:
            prompt[:] = prompt[0]
        start = prompt[:, cfg.kv_len].clone()
    else:
        for l in range(cfg.n_layers):
            kl, vl = synth.make_synthetic_kv(cfg, l, device=dev)
            if k.dtype == torch.uint8:   # the e4m3 codes of those values (exact)
                kl, vl = synth.fp8_kv_codes(kl, cfg.k_scale), synth.fp8_kv_codes(vl, cfg.v_scale)
            if pt is None:
                k[l, :, :, : cfg.kv_len] = kl
                v[l, :, :, : cfg.kv_len] = vl
            else:
                for b in range(B):
                    for t0 in range(0, cfg.kv_len, P):
                        t1 = min(t0 + P, cfg.kv_len)
                        pg = int(pt[b, t0 // P])
                        k[l, pg, :, : t1 - t0] = kl[b, :, t0:t1]
                        v[l, pg, :, : t1 - t0] = vl[b, :, t0:t1]
        start = synth.make_start_tokens(cfg, device="cpu")
    pt_dev = pt.to(dev) if pt is not None else None
    eng = Engine(cfg, w, k, v, n_ctas=n_ctas, spin_limit_us=spin_limit_us, flags=flags, window=window,
                 page_table=pt_dev, max_seq=ms if paged else None)
    m = GpuModel(cfg, w, k, v, eng, prompt, start.to(torch.int32), pt_dev)
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
