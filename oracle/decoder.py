"""Plain fp32 decoder forward on the CPU (test infrastructure; see oracle/__init__).

What one decode step computes.  The pages name the per-token operations of
decode without writing them out: attention QKV projection, softmax, activation,
normalisation and KV-cache update ("Persistent execution paradigm: from kernel
boundary elimination to ultra-low-latency engine", section 1), fused as
RMSNorm + projection (same page, section 5.3 and the TileRT fused-op list),
expert selection + gate/up + SiLU ("ExpertSelectUpGateSiLU", same page,
section 6) and greedy sampling inside the executed graph (same page, section 5.1).
The operations themselves follow the plain reading of a Llama-style decoder:

  x      = E[token]
  per layer:
    xn   = x * rsqrt(mean(x^2) + eps) * g_attn
    q,k,v = Wq xn, Wk xn, Wv xn
    q,k  = RoPE(q, pos), RoPE(k, pos)       rotate-half pairs (i, i + d/2)
    K[pos], V[pos] = bf16(k), bf16(v)
    o_h  = sum_t softmax_t(q_h . K_g[t] / sqrt(d)) V_g[t],  g = h // (n_q / n_kv), t in [0, pos]
    x   += Wo concat(o_h)
    xn2  = x * rsqrt(mean(x^2) + eps) * g_ffn
    dense: x += Wd (silu(Wg xn2) * Wu xn2)
    MoE:   p = softmax(Wr xn2); top-k of p (ties -> lower expert id);
           x += sum_e p_e FFN_e(xn2) + FFN_shared(xn2)
  logits = Wlm (x * rsqrt(mean(x^2) + eps) * g_final);  token = argmax (ties -> lowest id)

Everything is fp32 on the CPU except the KV cache, which stores bf16 like the
device cache (both sides round k and v to bf16 before attention reads them), or
for an e4m3 cache the e4m3 code of k / scale times a power-of-two scale per
tensor (kv_round).
The weights are widened from their stored bf16 / e4m3 bytes on use.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Tuple

import torch

from .fp4 import nvfp4_dequant
from .fp8 import e4m3_encode, e4m3_to_fp32


# --------------------------------------------------------------------------- ops

def rms_norm(x: torch.Tensor, g: torch.Tensor, eps: float) -> torch.Tensor:
    """x * rsqrt(mean(x^2) + eps) * g over the last axis, fp32."""
    x = x.float()
    ms = (x * x).mean(dim=-1, keepdim=True)
    return x * torch.rsqrt(ms + eps) * g.float()


def rope_angles(pos: int, head_dim: int, theta: float) -> Tuple[torch.Tensor, torch.Tensor]:
    """cos/sin of pos * theta^(-2i/d) for i < d/2, evaluated in fp64 and rounded to fp32."""
    i = torch.arange(head_dim // 2, dtype=torch.float64)
    inv = theta ** (-2.0 * i / head_dim)
    ang = float(pos) * inv
    return torch.cos(ang).float(), torch.sin(ang).float()


def rope_rotate(x: torch.Tensor, pos: int, theta: float) -> torch.Tensor:
    """Rotate-half RoPE of [..., heads, d] at position `pos`: pair (i, i+d/2) turns by pos*theta_i."""
    d = x.shape[-1]
    c, s = rope_angles(pos, d, theta)
    a, b = x[..., : d // 2], x[..., d // 2:]
    return torch.cat([a * c - b * s, a * s + b * c], dim=-1)


def attention_decode(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor) -> torch.Tensor:
    """Decode attention of one sequence.

    q [n_q][d] fp32; K, V [n_kv][T][d] (any float dtype, widened).  Query head h
    reads kv head h // (n_q / n_kv); scores are q.K/sqrt(d), softmax over all T
    positions (the new token's own entry included), output [n_q][d].
    """
    n_q, d = q.shape
    n_kv = K.shape[0]
    grp = n_q // n_kv
    out = torch.empty(n_q, d, dtype=torch.float32)
    for h in range(n_q):
        g = h // grp
        Kg, Vg = K[g].float(), V[g].float()
        s = (Kg @ q[h]) / math.sqrt(d)
        p = torch.softmax(s, dim=0)
        out[h] = p @ Vg
    return out


def silu(z: torch.Tensor) -> torch.Tensor:
    """z * sigmoid(z) = z / (1 + exp(-z))."""
    return z / (1.0 + torch.exp(-z))


def swiglu_ffn(xn: torch.Tensor, wg: torch.Tensor, wu: torch.Tensor, wd: torch.Tensor) -> torch.Tensor:
    """Wd (silu(Wg xn) * (Wu xn)) for one activation vector."""
    return wd @ (silu(wg @ xn) * (wu @ xn))


def moe_route(router_logits: torch.Tensor, k: int) -> Tuple[List[int], List[float], torch.Tensor]:
    """Softmax over all experts, then the k most probable (ties -> lower id), unrenormalised.

    Returns (ids, weights, probabilities).
    """
    p = torch.softmax(router_logits.float(), dim=0)
    order = sorted(range(p.numel()), key=lambda e: (-float(p[e]), e))
    ids = order[:k]
    return ids, [float(p[e]) for e in ids], p


def argmax_lowest(v: torch.Tensor) -> int:
    """Index of the maximum; the lowest index among equal maxima."""
    m = v.max()
    return int(torch.nonzero(v == m)[0, 0])


def _bf16_round(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def kv_round(x: torch.Tensor, kv_dtype: str, scale: float) -> torch.Tensor:
    """The value a cache entry holds: bf16 (round to nearest even), or for an
    e4m3 cache the code of x / scale (satfinite) times scale.  The scale is a
    power of two, so x / scale and code * scale are exact and the result is
    also exactly a bf16 value (4 significant bits)."""
    if kv_dtype == "bf16":
        return x.to(torch.bfloat16)
    assert kv_dtype == "fp8_e4m3" and scale > 0 and math.frexp(scale)[0] == 0.5, scale
    codes = e4m3_encode(x.float() / scale)
    return (e4m3_to_fp32(codes) * scale).to(torch.bfloat16)


# ------------------------------------------------------------------- the model

class OracleDecoder:
    """A seeded decoder held on the host, stepping one token per sequence per call.

    `weights` maps the names produced by synth.make_weights to host tensors.
    The KV cache is bf16 [L][B][n_kv][max_seq][d], K and V separately.
    """

    def __init__(self, cfg, weights: Dict[str, torch.Tensor], batch: Optional[int] = None,
                 max_seq: Optional[int] = None):
        self.cfg = cfg
        self.w = weights
        self.B = batch if batch is not None else cfg.batch
        self.max_seq = max_seq if max_seq is not None else cfg.max_seq
        shape = (cfg.n_layers, self.B, cfg.n_kv_heads, self.max_seq, cfg.head_dim)
        self.K = torch.zeros(shape, dtype=torch.bfloat16)
        self.V = torch.zeros(shape, dtype=torch.bfloat16)
        self.pos = [0] * self.B
        self.last_experts: List[List[List[int]]] = []

    # weights widened to fp32 on use
    def W(self, name: str) -> torch.Tensor:
        t = self.w[name]
        if t.dtype == torch.uint8 and (name + ".gscale") in self.w:
            # NVFP4: e2m1 codes, an e4m3 scale per 16 elements of a row, an fp32 tensor scale
            return nvfp4_dequant(t, self.w[name + ".scale"], float(self.w[name + ".gscale"].reshape(-1)[0]))
        if t.dtype == torch.uint8:
            sc = self.w[name + ".scale"]
            N, K = t.shape
            deq = e4m3_to_fp32(t).view(N // 128, 128, K // 128, 128) * sc[:, None, :, None]
            return deq.view(N, K)
        return t.float()

    def load_kv(self, layer: int, k: torch.Tensor, v: torch.Tensor) -> None:
        """Install cache contents [B][n_kv][T][d] at positions [0, T) of `layer`
        (values a cache of the model's KV type can hold: they are stored as given)."""
        T = k.shape[2]
        self.K[layer, :, :, :T] = k.to(torch.bfloat16)
        self.V[layer, :, :, :T] = v.to(torch.bfloat16)

    def _ffn(self, l: int, xn: torch.Tensor) -> Tuple[torch.Tensor, List[int]]:
        cfg = self.cfg
        p = f"layers.{l}."
        if not cfg.is_moe:
            return swiglu_ffn(xn, self.W(p + "w_gate"), self.W(p + "w_up"), self.W(p + "w_down")), []
        ids, gates, probs = moe_route(self.W(p + "router") @ xn, cfg.top_k)
        self._router_probs.append(probs)
        out = torch.zeros(cfg.hidden, dtype=torch.float32)
        for e, ge in zip(ids, gates):
            q = f"{p}experts.{e}."
            out += ge * swiglu_ffn(xn, self.W(q + "w_gate"), self.W(q + "w_up"), self.W(q + "w_down"))
        for s in range(cfg.n_shared_experts):
            q = f"{p}shared.{s}."
            out += swiglu_ffn(xn, self.W(q + "w_gate"), self.W(q + "w_up"), self.W(q + "w_down"))
        return out, ids

    def step(self, tokens: List[int]) -> Tuple[torch.Tensor, torch.Tensor]:
        """Feed token[b] at position pos[b] for every sequence; returns (logits [B][V], hidden [B][H]).

        `hidden` is the residual stream after the last layer (before the final norm).
        Appends one KV entry per layer per sequence and advances pos.
        """
        cfg = self.cfg
        d, nq, nkv = cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
        logits = torch.empty(self.B, cfg.vocab, dtype=torch.float32)
        hidden = torch.empty(self.B, cfg.hidden, dtype=torch.float32)
        experts: List[List[int]] = []
        self._router_probs: List[torch.Tensor] = []
        for b in range(self.B):
            pos = self.pos[b]
            assert pos < self.max_seq
            x = self.w["embed"][int(tokens[b])].float()
            for l in range(cfg.n_layers):
                p = f"layers.{l}."
                xn = rms_norm(x, self.w[p + "attn_norm"], cfg.rms_eps)
                q = (self.W(p + "wq") @ xn).view(nq, d)
                k = (self.W(p + "wk") @ xn).view(nkv, d)
                v = (self.W(p + "wv") @ xn).view(nkv, d)
                q = rope_rotate(q, pos, cfg.rope_theta)
                k = rope_rotate(k, pos, cfg.rope_theta)
                self.K[l, b, :, pos] = kv_round(k, cfg.kv_dtype, cfg.k_scale)
                self.V[l, b, :, pos] = kv_round(v, cfg.kv_dtype, cfg.v_scale)
                o = attention_decode(q, self.K[l, b, :, : pos + 1], self.V[l, b, :, : pos + 1])
                x = x + self.W(p + "wo") @ o.reshape(-1)
                xn2 = rms_norm(x, self.w[p + "ffn_norm"], cfg.rms_eps)
                f, ids = self._ffn(l, xn2)
                experts.append(ids)
                x = x + f
            hidden[b] = x
            logits[b] = self.W("lm_head") @ rms_norm(x, self.w["final_norm"], cfg.rms_eps)
            self.pos[b] = pos + 1
        self.last_experts = [experts[b * cfg.n_layers:(b + 1) * cfg.n_layers] for b in range(self.B)]
        # the router probabilities behind each selection (records only)
        self.last_router_probs = [self._router_probs[b * cfg.n_layers:(b + 1) * cfg.n_layers]
                                  for b in range(self.B)] if cfg.is_moe else []
        return logits, hidden

    # ---------------------------------------------------------------- prefill

    def forward_sequence(self, tokens: torch.Tensor, fill_cache: bool = True) -> torch.Tensor:
        """Full causal recompute over one prompt per sequence, from an empty cache.

        tokens int [B][T].  Every position attends to positions 0..t through a
        causal mask on the full score matrix (no cache is read).  Returns logits
        [B][T][V]; with fill_cache, writes bf16 K/V for positions [0, T) and sets
        pos = T.  Incremental decoding from position 0 must give the same result
        (the cache is only a memo of k and v).
        """
        cfg = self.cfg
        d, nq, nkv = cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
        grp = nq // nkv
        Bn, T = tokens.shape
        out = torch.empty(Bn, T, cfg.vocab, dtype=torch.float32)
        self._router_probs = []
        for b in range(Bn):
            x = self.w["embed"][tokens[b].long()].float()          # [T][H]
            for l in range(cfg.n_layers):
                p = f"layers.{l}."
                xn = rms_norm(x, self.w[p + "attn_norm"], cfg.rms_eps)
                q = (xn @ self.W(p + "wq").T).view(T, nq, d)
                k = (xn @ self.W(p + "wk").T).view(T, nkv, d)
                v = (xn @ self.W(p + "wv").T).view(T, nkv, d)
                qs, ks = torch.empty_like(q), torch.empty_like(k)
                for t in range(T):
                    qs[t] = rope_rotate(q[t], t, cfg.rope_theta)
                    ks[t] = rope_rotate(k[t], t, cfg.rope_theta)
                kb, vb = kv_round(ks, cfg.kv_dtype, cfg.k_scale), kv_round(v, cfg.kv_dtype, cfg.v_scale)
                if fill_cache:
                    self.K[l, b, :, :T] = kb.permute(1, 0, 2)
                    self.V[l, b, :, :T] = vb.permute(1, 0, 2)
                mask = torch.ones(T, T, dtype=torch.bool).tril()
                o = torch.empty(T, nq, d, dtype=torch.float32)
                for h in range(nq):
                    g = h // grp
                    s = (qs[:, h] @ kb[:, g].float().T) / math.sqrt(d)     # [T][T]
                    s = s.masked_fill(~mask, float("-inf"))
                    o[:, h] = torch.softmax(s, dim=1) @ vb[:, g].float()
                x = x + o.view(T, nq * d) @ self.W(p + "wo").T
                xn2 = rms_norm(x, self.w[p + "ffn_norm"], cfg.rms_eps)
                f = torch.stack([self._ffn(l, xn2[t])[0] for t in range(T)]) if cfg.is_moe else \
                    (silu(xn2 @ self.W(p + "w_gate").T) * (xn2 @ self.W(p + "w_up").T)) @ self.W(p + "w_down").T
                x = x + f
            out[b] = rms_norm(x, self.w["final_norm"], cfg.rms_eps) @ self.W("lm_head").T
            if fill_cache:
                self.pos[b] = T
        return out
