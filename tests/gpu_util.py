"""Helpers for the GPU parity tests: run the engine through the C ABI and replay
the same steps in the oracle (teacher-forced on the engine's emitted tokens)."""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

import synth
from oracle import OracleDecoder
from persistent_decode_b200 import workload

REL_L2_BF16 = 1e-2      # hidden-state and logit relative L2 tolerance (bf16 weights)
REL_L2_FP8 = 3e-2       # FP8 weights
ARGMAX_MARGIN = 1e-2    # argmax must agree where the oracle's top-2 gap exceeds this


@dataclasses.dataclass
class Run:
    tokens: torch.Tensor   # [n][B] int32 (host)
    logits: torch.Tensor   # [n][B][V] fp32 (host)
    hidden: torch.Tensor   # [n][B][H] fp32 (host)
    experts: Optional[torch.Tensor] = None   # MoE: [n][L][B][top_k] int32 (host)


ROUTER_GAP = 1e-6       # expert selections must match where the router probabilities differ by more


def run_engine(m: workload.GpuModel, n_steps: int, unfused: bool = False, keep_logits: bool = True) -> Run:
    cfg, dev = m.cfg, m.k.device
    B = cfg.batch
    workload.reset_state(m)
    tok = torch.empty(n_steps, B, dtype=torch.int32, device=dev)
    lg = torch.empty(n_steps, B, cfg.vocab, dtype=torch.float32, device=dev) if keep_logits else None
    hd = torch.empty(n_steps, B, cfg.hidden, dtype=torch.float32, device=dev)
    ex = torch.full((n_steps, cfg.n_layers, B, max(cfg.top_k, 1)), -1, dtype=torch.int32, device=dev) \
        if cfg.is_moe else None
    m.engine.decode(n_steps, tok, logits=lg, hidden=hd, experts=ex, unfused=unfused)
    m.engine.check()
    return Run(tok.cpu(), lg.cpu() if lg is not None else None, hd.cpu(), ex.cpu() if ex is not None else None)


def check_experts(run: Run, o: OracleDecoder, s: int, b: int) -> None:
    """Engine's expert choice at step s vs the oracle's last step: the selected set
    must agree wherever the k-th and (k+1)-th router probabilities differ by more
    than ROUTER_GAP, and the order wherever adjacent selected ones do."""
    cfg = o.cfg
    k = cfg.top_k
    for l in range(cfg.n_layers):
        probs = o.last_router_probs[b][l]
        ps = torch.sort(probs, descending=True).values
        got = [int(v) for v in run.experts[s, l, b, :k]]
        want = o.last_experts[b][l]
        boundary = float(ps[k - 1] - ps[k]) if k < probs.numel() else 1.0
        if boundary > ROUTER_GAP:
            assert sorted(got) == sorted(want), f"step {s} layer {l}: experts {got} != oracle {want}"
            if all(float(ps[i] - ps[i + 1]) > ROUTER_GAP for i in range(k - 1)):
                assert got == want, f"step {s} layer {l}: expert order {got} != oracle {want}"


class HostWeights(dict):
    """Host copies of the generator's weight tensors, fetched on first use.

    A large model's oracle touches only what it reads (a MoE step reads the
    router and the selected experts), so nothing else crosses to the host."""

    def __init__(self, dev_weights):
        super().__init__()
        self._src = dev_weights

    def __missing__(self, key):
        t = self._src[key].cpu()
        self[key] = t
        return t

    def __contains__(self, key):
        return key in self._src


class MemoOracle(OracleDecoder):
    """The oracle with each matrix widened (or FP8-dequantised) by its own W()
    once and kept in fp32, so that long replays do not redo the widening every
    step.  The arithmetic is the oracle's: W() itself produces the cached values."""

    def W(self, name: str) -> torch.Tensor:
        memo = self.__dict__.setdefault("_memo", {})
        t = memo.get(name)
        if t is None:
            t = super().W(name)
            memo[name] = t
            if isinstance(self.w, HostWeights):   # the fp32 copy replaces the stored bytes
                self.w.pop(name, None)
                self.w.pop(name + ".scale", None)
                self.w.pop(name + ".gscale", None)
        return t


def oracle_for(m: workload.GpuModel, max_seq: Optional[int] = None, memo: bool = False) -> OracleDecoder:
    """An oracle at the same decode start state as the engine.

    Weights are the generator's tensors, copied to the host as the oracle reads
    them.  Prompt workloads are prefilled by the oracle's own full causal
    recompute; synthetic-KV workloads get the generator's cache contents
    (regenerated, not read back from the engine's cache).  `memo` keeps each
    matrix's fp32 values after first use (long replays of large models).
    """
    cfg = m.cfg
    w = HostWeights(m.weights)
    cls = MemoOracle if memo else OracleDecoder
    o = cls(cfg, w, cfg.batch, max_seq=max_seq or m.engine.max_seq)
    if cfg.prefill:
        o.forward_sequence(m.prompt[:, : cfg.kv_len])
    else:
        dev = m.k.device
        for l in range(cfg.n_layers):
            kl, vl = synth.make_synthetic_kv(cfg, l, device=dev)
            o.load_kv(l, kl.cpu(), vl.cpu())
        o.pos = [cfg.kv_len] * cfg.batch
    return o


def rel_l2(a: torch.Tensor, b: torch.Tensor) -> float:
    return float((a.double() - b.double()).norm() / b.double().norm().clamp_min(1e-30))


def compare_with_oracle(m: workload.GpuModel, run: Run, o: OracleDecoder, n_check: int,
                        tol: float = REL_L2_BF16) -> List[dict]:
    """Teacher-forced replay of the first n_check steps; asserts the acceptance rules."""
    cfg = m.cfg
    report = []
    for s in range(n_check):
        inp = m.start_tokens.tolist() if s == 0 else run.tokens[s - 1].tolist()
        lg, hd = o.step(inp)
        for b in range(cfg.batch):
            e_h = rel_l2(run.hidden[s, b], hd[b])
            e_l = rel_l2(run.logits[s, b], lg[b]) if run.logits is not None else 0.0
            top2 = torch.topk(lg[b], 2)
            margin = float(top2.values[0] - top2.values[1])
            want = int(top2.indices[0])
            got = int(run.tokens[s, b])
            report.append(dict(step=s, b=b, hidden=e_h, logits=e_l, margin=margin, want=want, got=got))
            if run.experts is not None:
                check_experts(run, o, s, b)
            assert e_h <= tol, f"step {s} seq {b}: hidden rel L2 {e_h:.3e} > {tol}"
            assert e_l <= tol, f"step {s} seq {b}: logits rel L2 {e_l:.3e} > {tol}"
            if margin > ARGMAX_MARGIN:
                assert got == want, f"step {s} seq {b}: argmax {got} != oracle {want} (margin {margin:.3e})"
            else:
                # near-tie: the engine's token must be one of the oracle's top values within the margin
                assert float(lg[b, got]) >= float(top2.values[0]) - ARGMAX_MARGIN, (s, b, got)
    return report
