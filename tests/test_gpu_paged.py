"""Paged KV cache through the C ABI on a B200: the cache lives in a pool of
pages (one attention chunk each) scattered in a seeded random order, sequences
may share prefix pages, and the decode must equal the contiguous-cache decode
bit for bit (the same arithmetic on the same values), and the oracle."""
import pytest
import torch

import synth
from persistent_decode_b200 import XlpkError, _abi, workload

from tests.gpu_util import compare_with_oracle, oracle_for, run_engine

pytestmark = pytest.mark.gpu


def _same(a, b):
    assert torch.equal(a.tokens, b.tokens)
    assert torch.equal(a.logits, b.logits)
    assert torch.equal(a.hidden, b.hidden)


@pytest.mark.parametrize("unfused", [False, True], ids=["persistent", "kernel_per_op"])
def test_paged_cache_matches_contiguous(cuda_device, unfused):
    # two sequences with their own prompts (prefilled through the engine into the pages)
    cfg = synth.get_config("tiny", batch=2, steps=10)
    flat = workload.build(cfg, device=cuda_device, norm_std=0.1)
    paged = workload.build(cfg, device=cuda_device, norm_std=0.1, weights=flat.weights, paged=True)
    a = run_engine(flat, cfg.steps, unfused=unfused)
    b = run_engine(paged, cfg.steps, unfused=unfused)
    _same(a, b)
    n = cfg.kv_len + cfg.steps
    assert torch.equal(workload.contiguous_view(paged, "k")[:, :, :, :n], flat.k[:, :, :, :n])
    assert torch.equal(workload.contiguous_view(paged, "v")[:, :, :, :n], flat.v[:, :, :, :n])
    compare_with_oracle(paged, b, oracle_for(paged), cfg.steps)


def test_paged_head_dim_128_synthetic_cache(cuda_device):
    # d = 128 (64-position pages), a 200-position synthetic cache written into
    # the pages, ragged last page
    cfg = synth.get_config("tiny", hidden=512, n_q_heads=8, n_kv_heads=2, head_dim=128, ffn=1024, kv_len=200,
                           steps=8, batch=2, prefill=False)
    flat = workload.build(cfg, device=cuda_device, norm_std=0.1)
    paged = workload.build(cfg, device=cuda_device, norm_std=0.1, weights=flat.weights, paged=True)
    assert workload.page_size(cfg) == 64
    _same(run_engine(flat, cfg.steps), run_engine(paged, cfg.steps))


def test_shared_prefix_pages(cuda_device):
    # both sequences decode the same prompt; their first page (128 positions at
    # d = 64) is one pool page, written by both prefills with the same values
    cfg = synth.get_config("tiny", batch=2, kv_len=150, steps=8)
    own = workload.build(cfg, device=cuda_device, paged=True, same_prompt=True)
    shared = workload.build(cfg, device=cuda_device, weights=own.weights, paged=True, same_prompt=True,
                            shared_prefix_pages=1)
    assert int(shared.page_table[0, 0]) == int(shared.page_table[1, 0])
    a = run_engine(own, cfg.steps)
    b = run_engine(shared, cfg.steps)
    _same(a, b)
    assert torch.equal(b.tokens[:, 0], b.tokens[:, 1])


def test_page_outside_the_pool_is_reported(cuda_device):
    # a table entry past the pool is never followed: the decode stops with
    # XLPK_ERR_INVALID_ARG, and with the table repaired the handle decodes as before
    cfg = synth.get_config("tiny", steps=6)
    m = workload.build(cfg, device=cuda_device, paged=True, spin_limit_us=20000)
    ref = run_engine(m, cfg.steps)
    P = workload.page_size(cfg)
    j = (cfg.kv_len + 2) // P                        # the page a later step appends into
    good = int(m.page_table[0, j])
    m.page_table[0, j] = m.k.shape[1] + 5
    workload.reset_state(m)
    tok = torch.empty(cfg.steps, 1, dtype=torch.int32, device=cuda_device)
    m.engine.decode(cfg.steps, tok)
    with pytest.raises(XlpkError) as e:
        m.engine.check()
    assert e.value.status == _abi.XLPK_ERR_INVALID_ARG
    assert "page-table entry" in str(e.value)
    m.page_table[0, j] = good
    _same(run_engine(m, cfg.steps), ref)
