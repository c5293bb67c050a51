"""NVFP4 weights (e2m1 codes, an e4m3 scale per 16 elements of a row, an fp32
scale per matrix) vs the oracle, through the C ABI on a B200.

The GPU widens every code exactly, scales each 16-column partial sum by its
block scale and each row's sum by its matrix's scale, in fp32; the oracle
multiplies the decoded weights out and runs its fp32 forward.  So the two
agree up to fp32 summation order: hidden states and logits within the FP8
tolerance (3e-2 relative L2), the same greedy tokens where the top-2 margin is
clear.
"""
import pytest
import torch

import synth
from persistent_decode_b200 import workload
from persistent_decode_b200.engine import XlpkError

from tests.gpu_util import REL_L2_FP8, compare_with_oracle, oracle_for, run_engine

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("unfused", [False, True], ids=["persistent", "kernel_per_op"])
def test_tiny_nvfp4_matches_oracle(cuda_device, unfused):
    cfg = synth.get_config("tiny", weight_dtype="nvfp4", steps=10)
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, cfg.steps, unfused=unfused)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps, tol=REL_L2_FP8)


def test_nvfp4_head_dim_128_ragged_grid_with_gains(cuda_device):
    # d = 128, FFN 1536 (the down projection's K = 1536 is 3 chunks of 512), 37 CTAs
    cfg = synth.get_config("tiny", weight_dtype="nvfp4", hidden=512, n_q_heads=4, n_kv_heads=1,
                           head_dim=128, ffn=1536, kv_len=130, steps=6)
    m = workload.build(cfg, device=cuda_device, n_ctas=37, norm_std=0.1)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps, tol=REL_L2_FP8)


def test_nvfp4_batch2_is_refused(cuda_device):
    cfg = synth.get_config("tiny", weight_dtype="nvfp4", batch=2, steps=2)
    with pytest.raises(XlpkError, match="UNSUPPORTED"):
        workload.build(cfg, device=cuda_device)


def test_llama8b_nvfp4_full_size_prefix(cuda_device):
    # the 8B shape in NVFP4 (KV 8192, seeded synthetic cache): 4 steps against the oracle
    cfg = synth.get_config("llama8b_nvfp4", steps=4)
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m, memo=True), cfg.steps, tol=REL_L2_FP8)


def test_nvfp4_with_e4m3_cache(cuda_device):
    # both formats at once (their own kernel instantiation): NVFP4 weights, an e4m3 KV cache
    cfg = synth.fp8_kv(synth.get_config("tiny", weight_dtype="nvfp4", steps=8))
    m = workload.build(cfg, device=cuda_device)
    assert m.k.dtype == torch.uint8
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps, tol=REL_L2_FP8)
