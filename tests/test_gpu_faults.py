"""Failure detection on the GPU, without faulting it.

Every device-side wait of the persistent kernel is bounded.  These tests make
one wait run out on purpose -- CTA 0 withholds its release of one stage at the
call's first step (the withhold_release field of the decode call's io), so the waiters of the
next stage wait for a counter that never arrives -- and check that the kernel
ends on its own with XLPK_ERR_TIMEOUT reported through xlpk_get_status, that
every CTA left (the stream synchronises), and that the same handle decodes
correctly afterwards.
"""
import pytest
import torch

import synth
from persistent_decode_b200 import XlpkError, _abi, workload

from tests.gpu_util import run_engine

pytestmark = pytest.mark.gpu

SPIN_LIMIT_US = 20000   # 20 ms per wait keeps the failing calls short


@pytest.fixture(scope="module")
def tiny_fast_fail(cuda_device):
    cfg = synth.get_config("tiny", steps=8)
    return workload.build(cfg, device=cuda_device, spin_limit_us=SPIN_LIMIT_US)


# stage index = layer * 5 + kind (0 QKV, 2 O-proj, 3 gate/up, 4 down); the tiny
# bf16 model runs gate/up and down as one fused FFN stage (kind 3), so 8 is the
# last layer's FFN (its waiter is the LM head)
@pytest.mark.parametrize("stage", [0, 2, 3, 8])
def test_withheld_release_times_out_and_handle_recovers(tiny_fast_fail, stage):
    m = tiny_fast_fail
    ref = run_engine(m, 8)
    workload.reset_state(m)
    tok = torch.empty(8, 1, dtype=torch.int32, device=m.k.device)
    m.engine.decode(8, tok, withhold_release=stage + 1)
    with pytest.raises(XlpkError) as e:
        m.engine.check()
    assert e.value.status == _abi.XLPK_ERR_TIMEOUT
    assert "device wait failed" in str(e.value)
    # the status was reset with the counters: the handle works again
    again = run_engine(m, 8)
    assert torch.equal(again.tokens, ref.tokens)
    assert torch.equal(again.logits, ref.logits)
