"""An e4m3 KV cache (one power-of-two scale for K and one for V) against the
oracle, through the C ABI on a B200.

The oracle rounds every new K and V entry to the e4m3 code of x / scale
(round to nearest even, saturated) times the scale, exactly what the kernel's
QKV stage stores; the synthetic caches hold values on that grid.  So both
sides attend over the same cache values, except where a k or v lands within
rounding noise of a halfway point between two codes (a one-code difference).
Acceptance is the bf16 cache's: hidden state and logits within the relative-L2
tolerance and argmax equal wherever the oracle's top-2 margin exceeds 1e-2,
plus the cache's own entries against the oracle's.
"""
import pytest
import torch

import synth
from persistent_decode_b200 import workload

from tests.gpu_util import compare_with_oracle, oracle_for, rel_l2, run_engine

pytestmark = pytest.mark.gpu


def check_cache(m, o, T):
    """Cache entries [0, T) as values vs the oracle's.  Layer 0's k and v come
    from the embedding row alone (fp32 dot products in another order), so they
    differ at most where a value sits within rounding noise of a halfway point:
    one e4m3 step.  Later layers see the small upstream differences of the two
    decodes, so a small entry may move a few of its own steps; those are bounded
    against the tensor's RMS."""
    for which, ref, scale in (("k", o.K, m.cfg.k_scale), ("v", o.V, m.cfg.v_scale)):
        got = workload.kv_values(m, which)[:, :, :, :T].float().cpu()
        want = ref[:, :, :, :T].float()
        differ = got != want
        assert float(differ.float().mean()) < 1e-3, which
        # e4m3 keeps 4 significant bits: neighbouring values are <= 1/8 apart relatively
        d0 = (got[0] - want[0]).abs()[differ[0]]
        assert bool((d0 <= want[0].abs()[differ[0]] / 8 + 2.0 ** -9 * scale).all()), which
        rms = float(want.pow(2).mean().sqrt())
        d = (got - want).abs()[differ]
        assert bool((d <= want.abs()[differ] / 8 + 1e-3 * rms + 2.0 ** -9 * scale).all()), which
        assert rel_l2(got, want) < 1e-2, which


def test_tiny_fp8_kv_prompt(cuda_device):
    # d = 64 (chunks of 128 positions): a 128-token prompt prefilled through the
    # engine into the e4m3 cache, then 16 greedy steps
    cfg = synth.fp8_kv(synth.get_config("tiny", steps=16))
    m = workload.build(cfg, device=cuda_device)
    assert m.k.dtype == torch.uint8
    run = run_engine(m, cfg.steps)
    o = oracle_for(m)
    compare_with_oracle(m, run, o, cfg.steps)
    check_cache(m, o, cfg.kv_len + cfg.steps)


@pytest.mark.parametrize("unfused", [False, True])
def test_d128_fp8_kv_ragged(cuda_device, unfused):
    # d = 128 (chunks of 64 positions), 200 prompt positions = 3 chunks + 8
    cfg = synth.fp8_kv(synth.get_config("tiny", hidden=512, n_q_heads=4, n_kv_heads=1, head_dim=128,
                                        ffn=1024, kv_len=200, steps=10))
    m = workload.build(cfg, device=cuda_device, norm_std=0.1)
    run = run_engine(m, cfg.steps, unfused=unfused)
    o = oracle_for(m)
    compare_with_oracle(m, run, o, cfg.steps)
    check_cache(m, o, cfg.kv_len + cfg.steps)


@pytest.mark.parametrize("batch", [2, 8])
def test_fp8_kv_synthetic_cache_batches(cuda_device, batch):
    # a seeded synthetic e4m3 cache of 1000 positions (7 chunks + 104) per
    # sequence at d = 128, several sequences decoded together
    cfg = synth.fp8_kv(synth.get_config("tiny", hidden=512, n_q_heads=8, n_kv_heads=2, head_dim=128,
                                        ffn=1024, kv_len=1000, steps=6, batch=batch, prefill=False))
    m = workload.build(cfg, device=cuda_device, norm_std=0.1)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps)


def test_fp8_kv_paged(cuda_device):
    # the e4m3 cache in a scattered page pool (a page is one chunk: 64 positions
    # of d = 128, 8 KB of codes per K or V page) gives the contiguous cache's tokens
    cfg = synth.fp8_kv(synth.get_config("tiny", hidden=512, n_q_heads=4, n_kv_heads=2, head_dim=128,
                                        ffn=1024, kv_len=300, steps=8, batch=2, prefill=False))
    flat = workload.build(cfg, device=cuda_device, norm_std=0.1)
    paged = workload.build(cfg, device=cuda_device, norm_std=0.1, paged=True, weights=flat.weights)
    assert paged.k.dtype == torch.uint8
    rf = run_engine(flat, cfg.steps)
    rp = run_engine(paged, cfg.steps)
    assert torch.equal(rf.tokens, rp.tokens)
    n = cfg.kv_len + cfg.steps
    assert torch.equal(workload.contiguous_view(paged, "k")[:, :, :, :n], flat.k[:, :, :, :n])
    compare_with_oracle(paged, rp, oracle_for(paged), cfg.steps)


def test_fp8_kv_saturates(cuda_device):
    # a K scale so small that most new entries exceed 448 codes: the kernel
    # stores +-448 (satfinite), as the oracle does
    cfg = synth.get_config("tiny", steps=4).with_(kv_dtype="fp8_e4m3", k_scale=2.0 ** -12, v_scale=2.0 ** -6)
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, cfg.steps)
    o = oracle_for(m)
    compare_with_oracle(m, run, o, cfg.steps)
    T = cfg.kv_len + cfg.steps
    codes = m.k[:, :, :, :T].cpu()
    sat = (codes & 0x7F) == 0x7E                     # +-448
    assert float(sat.float().mean()) > 0.01
    assert not bool(((codes & 0x7F) == 0x7F).any())  # never NaN
    check_cache(m, o, T)


def test_llama8b_fp8_kv_full_size(cuda_device):
    # the headline shape with an e4m3 cache: 8192 cached positions (seeded
    # synthetic e4m3 cache), 8 greedy steps in one launch
    cfg = synth.fp8_kv(synth.get_config("llama8b", steps=8))
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m, memo=True), cfg.steps)
