"""MoE decode (router, top-k routing, shared + routed SwiGLU experts) vs the
oracle, through the C ABI on a B200: hidden states and logits within the bf16
tolerance, the same greedy tokens where the top-2 margin is clear, and the same
expert selection wherever the router probabilities separate by more than 1e-6."""
import pytest
import torch

import synth
from persistent_decode_b200 import workload

from tests.gpu_util import compare_with_oracle, oracle_for, run_engine

pytestmark = pytest.mark.gpu


def _moe_cfg(**kw):
    base = dict(n_experts=8, top_k=2, n_shared_experts=1, expert_ffn=128, ffn=0, steps=8)
    base.update(kw)
    return synth.get_config("tiny", **base)


@pytest.mark.parametrize("unfused", [False, True], ids=["persistent", "kernel_per_op"])
def test_tiny_moe_matches_oracle(cuda_device, unfused):
    # prompt prefill through the engine exercises the routing at every position
    cfg = _moe_cfg()
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, cfg.steps, unfused=unfused)
    assert int(run.experts.min()) >= 0 and int(run.experts.max()) < cfg.n_experts
    compare_with_oracle(m, run, oracle_for(m), cfg.steps)


def test_moe_persistent_equals_kernel_per_op(cuda_device):
    cfg = _moe_cfg(steps=6)
    m = workload.build(cfg, device=cuda_device)
    a = run_engine(m, cfg.steps)
    b = run_engine(m, cfg.steps, unfused=True)
    assert torch.equal(a.tokens, b.tokens)
    assert torch.equal(a.experts, b.experts)
    assert torch.equal(a.logits, b.logits)


def test_moe_wider_shape_and_gains(cuda_device):
    # head_dim 128 with 4-query-head groups (the MoE workload's attention),
    # 16 experts, top-4, two shared experts, expert width 256, a KV length that
    # spans several chunks with a ragged tail, non-unit norm gains
    cfg = _moe_cfg(hidden=512, n_q_heads=8, n_kv_heads=2, head_dim=128, n_experts=16, top_k=4,
                   n_shared_experts=2, expert_ffn=256, kv_len=150, steps=6)
    m = workload.build(cfg, device=cuda_device, norm_std=0.1)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps)


def test_moe_ragged_grid_no_shared(cuda_device):
    # a grid that divides nothing evenly and no shared expert
    cfg = _moe_cfg(n_shared_experts=0, top_k=3, steps=5)
    m = workload.build(cfg, device=cuda_device, n_ctas=37)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps)
