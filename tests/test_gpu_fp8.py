"""FP8 (e4m3, one fp32 scale per 128x128 block) weights vs the oracle, through
the C ABI on a B200: hidden states and logits within the FP8 tolerance (3e-2
relative L2), the same greedy tokens where the top-2 margin is clear."""
import pytest
import torch

import synth
from persistent_decode_b200 import workload

from tests.gpu_util import REL_L2_FP8, compare_with_oracle, oracle_for, run_engine

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("unfused", [False, True], ids=["persistent", "kernel_per_op"])
def test_tiny_fp8_matches_oracle(cuda_device, unfused):
    cfg = synth.get_config("tiny", weight_dtype="fp8_e4m3", steps=10)
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, cfg.steps, unfused=unfused)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps, tol=REL_L2_FP8)


@pytest.mark.parametrize("batch", [2, 4])
def test_tiny_fp8_batched_with_gains(cuda_device, batch):
    cfg = synth.get_config("tiny", weight_dtype="fp8_e4m3", batch=batch, steps=6)
    m = workload.build(cfg, device=cuda_device, norm_std=0.1)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps, tol=REL_L2_FP8)


def test_fp8_head_dim_128_ragged_grid(cuda_device):
    # d = 128 with 4-query-head groups, FFN 1024 (down K spans chunks), 37 CTAs
    cfg = synth.get_config("tiny", weight_dtype="fp8_e4m3", hidden=512, n_q_heads=4, n_kv_heads=1,
                           head_dim=128, ffn=1024, kv_len=130, steps=6)
    m = workload.build(cfg, device=cuda_device, n_ctas=37)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps, tol=REL_L2_FP8)


def test_llama8b_fp8_full_size_prefix(cuda_device):
    # the 8B shape with block-scaled FP8 weights and its 1024-entry synthetic
    # cache, in the launch configuration the bench times
    cfg = synth.get_config("llama8b_fp8")
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, 8)
    o = oracle_for(m)
    compare_with_oracle(m, run, o, 2, tol=REL_L2_FP8)
    assert int(run.tokens.min()) >= 0 and int(run.tokens.max()) < cfg.vocab


def test_llama8b_fp8_batch2_full_size_prefix(cuda_device):
    # the 8B FP8 shape at batch 2 (two sequences over the 1024-entry synthetic
    # cache); its activation region holds 2 x 14336 floats, so the ring keeps
    # 3 slots
    cfg = synth.get_config("llama8b_fp8", batch=2)
    m = workload.build(cfg, device=cuda_device)
    assert m.engine.info().ring_slots >= 2
    run = run_engine(m, 4)
    compare_with_oracle(m, run, oracle_for(m), 2, tol=REL_L2_FP8)
    assert int(run.tokens.min()) >= 0 and int(run.tokens.max()) < cfg.vocab


@pytest.mark.parametrize("batch", [4, 8])
def test_llama8b_fp8_large_batch_full_size_prefix(cuda_device, batch):
    # the 8B FP8 shape at batch 4 and 8: B x 14336 fp32 down-projection inputs
    # do not fit beside the ring, so W_down streams in K windows of 4096
    cfg = synth.get_config("llama8b_fp8", batch=batch)
    m = workload.build(cfg, device=cuda_device)
    assert m.engine.info().ring_slots >= 2
    run = run_engine(m, 3)
    compare_with_oracle(m, run, oracle_for(m), 2, tol=REL_L2_FP8)


def test_tiny_fp8_batch8_tensor_core(cuda_device):
    # FP8 tiles widened to bf16 in their ring slot before the MMA
    cfg = synth.get_config("tiny", weight_dtype="fp8_e4m3", batch=8, steps=6)
    m = workload.build(cfg, device=cuda_device, norm_std=0.1)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps, tol=REL_L2_FP8)
