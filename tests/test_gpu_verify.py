"""Speculative verification (one launch checks k drafted tokens and accepts the
longest correct prefix on the device) through the C ABI on a B200: the emitted
tokens must be exactly the greedy decode's, and the per-position argmaxes and
logits must match the oracle fed the same tokens."""
import pytest
import torch

import synth
from persistent_decode_b200 import workload

from tests.gpu_util import REL_L2_BF16, oracle_for, rel_l2, run_engine

pytestmark = pytest.mark.gpu


def _verifier(cfg, k, dev, weights):
    # batch k + 1 sharing every page: one sequence seen at k + 1 consecutive positions
    vcfg = cfg.with_(batch=k + 1)
    P = workload.page_size(vcfg)
    pages = (vcfg.max_seq + P - 1) // P
    return workload.build(vcfg, device=dev, weights=weights, paged=True, same_prompt=True,
                          shared_prefix_pages=pages, spare_pages=0)


@pytest.mark.parametrize("k", [1, 3, 7])
def test_verify_emits_the_greedy_tokens(cuda_device, k):
    cfg = synth.get_config("tiny", steps=40)
    ref_model = workload.build(cfg, device=cuda_device)
    greedy = run_engine(ref_model, 24).tokens[:, 0].tolist()   # greedy continuation after the prompt
    v = _verifier(cfg, k, cuda_device, ref_model.weights)
    workload.reset_state(v)
    dev = cuda_device
    out, pos = [], 0
    argmax = torch.empty(k + 1, dtype=torch.int32, device=dev)
    wrong_at = [k - 1, k, 0, k]          # draft index made wrong in each call (k: all correct)
    for call in range(4):
        drafts = list(greedy[pos:pos + k])
        j = wrong_at[call]
        if j < k:
            drafts[j] = (drafts[j] + 1) % cfg.vocab
        n = v.engine.verify(torch.tensor(drafts, dtype=torch.int32, device=dev), argmax)
        assert n == (j + 1 if j < k else k + 1)
        out += greedy[pos:pos + n]
        emitted = drafts[:n - 1] + [int(argmax[n - 1])]
        assert emitted == greedy[pos:pos + n]
        pos += n
    assert len(out) == pos


def test_verify_logits_match_the_oracle(cuda_device):
    # each position's logits against the oracle fed the same tokens (teacher-forced)
    k = 3
    cfg = synth.get_config("tiny", steps=16)
    base = workload.build(cfg, device=cuda_device, norm_std=0.1)
    greedy = run_engine(base, 8).tokens[:, 0].tolist()
    v = _verifier(cfg, k, cuda_device, base.weights)
    workload.reset_state(v)
    drafts = greedy[:k]
    drafts[1] = (drafts[1] + 7) % cfg.vocab       # accept 1 draft + bonus
    argmax = torch.empty(k + 1, dtype=torch.int32, device=cuda_device)
    lg = torch.empty(1, k + 1, cfg.vocab, dtype=torch.float32, device=cuda_device)
    n = v.engine.verify(torch.tensor(drafts, dtype=torch.int32, device=cuda_device), argmax, logits=lg)
    assert n == 2
    o = oracle_for(base)
    fed = [int(base.start_tokens[0])] + drafts
    for i, t in enumerate(fed):
        ref, _ = o.step([t])
        assert rel_l2(lg[0, i].cpu(), ref[0]) <= REL_L2_BF16
        top2 = torch.topk(ref[0], 2)
        if float(top2.values[0] - top2.values[1]) > 1e-2:
            assert int(argmax[i]) == int(top2.indices[0])
