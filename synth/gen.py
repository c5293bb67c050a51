"""Counter-based seeded generators (host or CUDA, bit-identical).

Every random value is a pure function of (seed, stream name, element index):

* stream key   k = mix64(seed ^ FNV-1a-64(name))
* raw draw     r_i = mix64(k + (i + 1) * 0x9E3779B97F4A7C15)   (mod 2^64)

where mix64 is the SplitMix64 output function (Steele, Lea & Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014): three xor-shift /
multiply rounds with the published constants.  A normal draw uses the two
32-bit halves of r_i as open-interval uniforms and the Box-Muller transform
(fp64), then rounds to fp32 and to bf16 (round-to-nearest-even) with integer
arithmetic only, so the CPU and CUDA versions of this code agree bit for bit
except where a libm and the CUDA fp64 log/cos differ in the last fp64 ulp
exactly at a bf16 rounding boundary (probability ~2^-44 per element).

All arithmetic here uses torch int64 tensors (two's-complement wrap-around
multiplication; logical right shifts are masked explicitly), so the same code
runs on the host for the oracle and on a GPU for the CUDA path's inputs.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import torch

from .configs import DecoderConfig

_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_CHUNK = 1 << 23


def _s64(v: int) -> int:
    """Reinterpret an unsigned 64-bit integer as int64."""
    v &= (1 << 64) - 1
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix64_int(z: int) -> int:
    z &= (1 << 64) - 1
    z = ((z ^ (z >> 30)) * _M1) & ((1 << 64) - 1)
    z = ((z ^ (z >> 27)) * _M2) & ((1 << 64) - 1)
    return z ^ (z >> 31)


def _fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for b in name.encode():
        h ^= b
        h = (h * 0x100000001B3) & ((1 << 64) - 1)
    return h


def stream_key(seed: int, name: str) -> int:
    return _mix64_int((seed & ((1 << 64) - 1)) ^ _fnv1a64(name))


def _lsr(x: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 holding a uint64 bit pattern."""
    return (x >> k) & ((1 << (64 - k)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def splitmix64_stream(seed: int, name: str, start: int, n: int,
                      device: torch.device | str = "cpu") -> torch.Tensor:
    """Raw 64-bit draws r_start .. r_{start+n-1} of stream (seed, name) as int64 bit patterns."""
    key = stream_key(seed, name)
    idx = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = idx * _s64(_GAMMA) + _s64(key)
    return _mix64(z)


def _fp32_to_bf16_bits(x32: torch.Tensor) -> torch.Tensor:
    """fp32 -> bf16 round-to-nearest-even on the bit pattern (inputs are finite)."""
    b = x32.view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    lsb = (b >> 16) & 1
    r = (b + 0x7FFF + lsb) >> 16
    r = r & 0xFFFF
    return torch.where(r >= 0x8000, r - 0x10000, r).to(torch.int16)


def _normals_fp64(raw: torch.Tensor) -> torch.Tensor:
    hi = _lsr(raw, 32).to(torch.float64)
    lo = (raw & 0xFFFFFFFF).to(torch.float64)
    u1 = (hi + 0.5) * (1.0 / 4294967296.0)
    u2 = (lo + 0.5) * (1.0 / 4294967296.0)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def normal_fp32(seed: int, name: str, shape, std: float, mean: float = 0.0,
                device: torch.device | str = "cpu") -> torch.Tensor:
    """N(mean, std^2) draws of stream (seed, name), rounded once from fp64 to fp32."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.float32, device=device)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        z = _normals_fp64(splitmix64_stream(seed, name, s, m, device))
        out[s:s + m] = (z * std + mean).to(torch.float32)
    return out.view(*shape)


def normal_bf16(seed: int, name: str, shape, std: float,
                device: torch.device | str = "cpu") -> torch.Tensor:
    """N(0, std^2) draws rounded fp64 -> fp32 -> bf16 (RNE), as a bfloat16 tensor."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.int16, device=device)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        z = _normals_fp64(splitmix64_stream(seed, name, s, m, device))
        out[s:s + m] = _fp32_to_bf16_bits((z * std).to(torch.float32))
    return out.view(torch.bfloat16).view(*shape)


def uniform_tokens(seed: int, name: str, shape, vocab: int,
                   device: torch.device | str = "cpu") -> torch.Tensor:
    """Token ids uniform on [0, vocab) via a 32x32 multiply-shift of the draw's high half."""
    n = math.prod(shape)
    raw = splitmix64_stream(seed, name, 0, n, device)
    hi = _lsr(raw, 32)
    return ((hi * vocab) >> 32).to(torch.int32).view(*shape)


FP8_E4M3_MAX = 448.0


def quantize_fp8_blocks(w: torch.Tensor, block: int = 128):
    """Block-scaled e4m3 quantisation of a [N][K] weight (input preparation only).

    Per 128x128 block: scale = max|w| / 448 (1 for an all-zero block) and
    codes = e4m3(w / scale) with round-to-nearest-even, clamped to +-448.
    Returns (codes uint8 [N][K], scales fp32 [N/128][K/128]).
    """
    N, K = w.shape
    assert N % block == 0 and K % block == 0
    wf = w.float().view(N // block, block, K // block, block)
    amax = wf.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / FP8_E4M3_MAX, torch.ones_like(amax))
    q = (wf / scale[:, None, :, None]).clamp(-FP8_E4M3_MAX, FP8_E4M3_MAX)
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8).view(N, K)
    return codes.contiguous(), scale.contiguous()


FP4_E2M1_MAX = 6.0
_E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)   # codes 0..7


def quantize_nvfp4(w: torch.Tensor):
    """NVFP4 quantisation of a [N][K] weight (input preparation only).

    Tensor scale gs = max|w| / (448 * 6) (1 for an all-zero tensor); per 16
    consecutive elements of a row, block scale = e4m3(max|block| / (6 gs))
    (round to nearest even); codes = the E2M1 magnitude nearest to
    |w| / (block scale * gs) (ties to the even code, saturated at 6) with w's
    sign; an all-zero block gets scale 0 and codes 0.  Returns (codes uint8
    [N][K/2] with element 2j in the low nibble, block scales uint8 e4m3 codes
    [N][K/16], tensor scale fp32 [1]).
    """
    N, K = w.shape
    assert K % 16 == 0
    wf = w.float()
    amax = float(wf.abs().max())
    gs = amax / (FP8_E4M3_MAX * FP4_E2M1_MAX) if amax > 0 else 1.0
    blocks = wf.view(N, K // 16, 16)
    bmax = blocks.abs().amax(dim=-1)
    sb = (bmax / (FP4_E2M1_MAX * gs)).clamp(max=FP8_E4M3_MAX).to(torch.float8_e4m3fn)
    s = (sb.float() * gs)[..., None]
    y = torch.where(s > 0, blocks / torch.where(s > 0, s, torch.ones_like(s)), torch.zeros_like(blocks))
    mags = torch.tensor(_E2M1_MAGNITUDES, dtype=torch.float32, device=w.device)
    a = y.abs().clamp(max=FP4_E2M1_MAX)
    hi = torch.searchsorted(mags, a.contiguous()).clamp(max=7)
    lo = (hi - 1).clamp(min=0)
    d_hi, d_lo = mags[hi] - a, a - mags[lo]
    take_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0) & (lo != hi))
    code = torch.where(take_lo, lo, hi) | ((y < 0).to(torch.int64) << 3)
    code = code.view(N, K // 2, 2)
    packed = (code[..., 0] | (code[..., 1] << 4)).to(torch.uint8)
    return packed.contiguous(), sb.view(torch.uint8).contiguous(), torch.tensor([gs], dtype=torch.float32,
                                                                                 device=w.device)


def _linear(cfg: DecoderConfig, name: str, n: int, k: int, device, out: Dict[str, torch.Tensor]):
    w = normal_bf16(cfg.seed, name, (n, k), cfg.init_std, device)
    if cfg.weight_dtype == "fp8_e4m3":
        codes, scales = quantize_fp8_blocks(w)
        out[name] = codes
        out[name + ".scale"] = scales
    elif cfg.weight_dtype == "nvfp4":
        codes, scales, gs = quantize_nvfp4(w)
        out[name] = codes
        out[name + ".scale"] = scales
        out[name + ".gscale"] = gs
    else:
        out[name] = w


def _gain(cfg: DecoderConfig, name: str, n: int, norm_std: float, device) -> torch.Tensor:
    if norm_std == 0.0:
        return torch.ones(n, dtype=torch.float32, device=device)
    return normal_fp32(cfg.seed, name, (n,), norm_std, mean=1.0, device=device)


def make_weights(cfg: DecoderConfig, device: torch.device | str = "cpu",
                 norm_std: float = 0.0, layers: Optional[range] = None,
                 lm_head: bool = True) -> Dict[str, torch.Tensor]:
    """Row-major ([out][in]) random-init weights of `cfg`, keyed by name.

    Linear and embedding matrices are N(0, init_std^2) in bf16 (block-scaled
    e4m3 codes plus fp32 scales for the FP8 workload; the embedding and the
    MoE router stay bf16).  Norm gains are 1 (norm_std = 0) or 1 + N(0, norm_std^2).
    `layers` restricts generation to a subset (a bounded sample of a large model).
    """
    H, F = cfg.hidden, cfg.ffn
    w: Dict[str, torch.Tensor] = {}
    w["embed"] = normal_bf16(cfg.seed, "embed", (cfg.vocab, H), cfg.init_std, device)
    if lm_head:
        _linear(cfg, "lm_head", cfg.vocab, H, device, w)
        w["final_norm"] = _gain(cfg, "final_norm", H, norm_std, device)
    for l in (layers if layers is not None else range(cfg.n_layers)):
        p = f"layers.{l}."
        w[p + "attn_norm"] = _gain(cfg, p + "attn_norm", H, norm_std, device)
        w[p + "ffn_norm"] = _gain(cfg, p + "ffn_norm", H, norm_std, device)
        _linear(cfg, p + "wq", cfg.q_dim, H, device, w)
        _linear(cfg, p + "wk", cfg.kv_dim, H, device, w)
        _linear(cfg, p + "wv", cfg.kv_dim, H, device, w)
        _linear(cfg, p + "wo", H, cfg.q_dim, device, w)
        if cfg.is_moe:
            Fe, E = cfg.expert_ffn, cfg.n_experts
            w[p + "router"] = normal_bf16(cfg.seed, p + "router", (E, H), cfg.init_std, device)
            for e in range(E):
                q = f"{p}experts.{e}."
                _linear(cfg, q + "w_gate", Fe, H, device, w)
                _linear(cfg, q + "w_up", Fe, H, device, w)
                _linear(cfg, q + "w_down", H, Fe, device, w)
            for s in range(cfg.n_shared_experts):
                q = f"{p}shared.{s}."
                _linear(cfg, q + "w_gate", Fe, H, device, w)
                _linear(cfg, q + "w_up", Fe, H, device, w)
                _linear(cfg, q + "w_down", H, Fe, device, w)
        else:
            _linear(cfg, p + "w_gate", F, H, device, w)
            _linear(cfg, p + "w_up", F, H, device, w)
            _linear(cfg, p + "w_down", H, F, device, w)
    return w


def make_prompt(cfg: DecoderConfig, device: torch.device | str = "cpu") -> torch.Tensor:
    """Seeded random prompts, int32 [B][kv_len + 1]; sequence b uses seed 1 + b."""
    rows = [uniform_tokens(1 + b, "prompt", (cfg.kv_len + 1,), cfg.vocab, device)
            for b in range(cfg.batch)]
    return torch.stack(rows, 0)


def make_synthetic_kv(cfg: DecoderConfig, layer: int, device: torch.device | str = "cpu"):
    """Seeded synthetic cache contents for one layer: K and V bf16 [B][n_kv][kv_len][d].

    Entries are N(0, (init_std * sqrt(hidden))^2), the spread a projection of a
    unit-RMS activation through N(0, init_std^2) weights would give.
    """
    std = cfg.init_std * math.sqrt(cfg.hidden)
    shape = (cfg.batch, cfg.n_kv_heads, cfg.kv_len, cfg.head_dim)
    k = normal_bf16(2, f"kv.k.{layer}", shape, std, device)
    v = normal_bf16(2, f"kv.v.{layer}", shape, std, device)
    if cfg.kv_dtype == "fp8_e4m3":
        # values an e4m3 cache holds (code x power-of-two scale), still as bf16
        k = fp8_kv_values(k, cfg.k_scale)
        v = fp8_kv_values(v, cfg.v_scale)
    return k, v


def fp8_kv_values(x: torch.Tensor, scale: float) -> torch.Tensor:
    """Synthetic entries of an e4m3 cache (input preparation): x / scale rounded to
    e4m3 (satfinite, round to nearest even), times scale, as bf16 (exact)."""
    q = (x.float() / scale).clamp(-FP8_E4M3_MAX, FP8_E4M3_MAX).to(torch.float8_e4m3fn)
    return (q.float() * scale).to(torch.bfloat16)


def fp8_kv_codes(x: torch.Tensor, scale: float) -> torch.Tensor:
    """The uint8 e4m3 codes of cache values x that fp8_kv_values produced (exact)."""
    return (x.float() / scale).clamp(-FP8_E4M3_MAX, FP8_E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)


def make_start_tokens(cfg: DecoderConfig, device: torch.device | str = "cpu") -> torch.Tensor:
    """Pending token per sequence for the synthetic-KV workloads, int32 [B]."""
    return uniform_tokens(3, "start", (cfg.batch,), cfg.vocab, device)
