"""The device-resident request loop (serve mode) through the C ABI on a B200:
one launch stays resident while the host posts requests; every request's
tokens must equal those of ordinary decode calls from the same state, and the
loop must leave on its own when idle and come back on the next request."""
import time

import pytest
import torch

import synth
from persistent_decode_b200 import XlpkError, _abi, workload

from tests.gpu_util import run_engine

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny2(cuda_device):
    return workload.build(synth.get_config("tiny", batch=2, steps=24), device=cuda_device)


def test_requests_in_one_launch_match_decode(tiny2):
    m = tiny2
    ref = run_engine(m, 16)                           # 16 steps from the start state
    workload.reset_state(m)
    m.engine.serve_start(idle_limit_us=2_000_000)
    try:
        got = []
        for n in (5, 3, 8):                           # one request at a time
            first = m.engine.serve_post(n)
            got += m.engine.serve_wait(first, n)
    finally:
        m.engine.serve_stop()
    assert torch.equal(torch.tensor(got, dtype=torch.int32), ref.tokens)
    # the session's steps are part of the handle's state: a decode continues after them
    tok = torch.empty(4, 2, dtype=torch.int32, device=m.k.device)
    m.engine.decode(4, tok)
    m.engine.check()
    ref20 = run_engine(m, 20)
    assert torch.equal(tok.cpu(), ref20.tokens[16:20])


def test_requests_posted_ahead(tiny2):
    m = tiny2
    ref = run_engine(m, 12)
    workload.reset_state(m)
    m.engine.serve_start(idle_limit_us=2_000_000)
    try:
        firsts = [m.engine.serve_post(n) for n in (4, 4, 4)]   # queued before any wait
        got = []
        for f in firsts:
            got += m.engine.serve_wait(f, 4)
    finally:
        m.engine.serve_stop()
    assert torch.equal(torch.tensor(got, dtype=torch.int32), ref.tokens)


def test_idle_loop_leaves_and_comes_back(tiny2):
    m = tiny2
    ref = run_engine(m, 6)
    workload.reset_state(m)
    m.engine.serve_start(idle_limit_us=20_000)            # 20 ms without a request: leave
    try:
        got = m.engine.serve_wait(m.engine.serve_post(3), 3)
        time.sleep(0.3)                                    # the loop has left meanwhile
        torch.cuda.synchronize()
        got += m.engine.serve_wait(m.engine.serve_post(3), 3)   # launched again, same session
    finally:
        m.engine.serve_stop()
    assert torch.equal(torch.tensor(got, dtype=torch.int32), ref.tokens)


def test_handle_is_owned_by_the_session(tiny2):
    m = tiny2
    workload.reset_state(m)
    m.engine.serve_start(idle_limit_us=2_000_000)
    try:
        tok = torch.empty(2, 2, dtype=torch.int32, device=m.k.device)
        with pytest.raises(XlpkError) as e:
            m.engine.decode(2, tok)
        assert e.value.status == _abi.XLPK_ERR_INVALID_ARG
        with pytest.raises(XlpkError):
            m.engine.serve_post(10_000)                   # past max_seq
    finally:
        m.engine.serve_stop()
