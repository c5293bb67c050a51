"""xlpk_decode_noalloc: the allocation-free decode entry point.

Some callers must not allocate device memory while they decode (graph capture,
threads that must stay out of the CUDA allocator, memory owned by another
framework's allocator).  For them the library keeps the decode kernel's scratch
in a fixed array of its own; these tests check, through the C ABI, that this
variant gives the same results as xlpk_decode on two calls in a row, and that a
handle whose scratch does not fit is refused with a clear error.  The file is
named so that pytest collects it last.
"""
import ctypes as C

import pytest
import torch

import synth
from persistent_decode_b200 import XlpkError, _abi, get_lib, workload

from tests.gpu_util import REL_L2_BF16, rel_l2, run_engine

pytestmark = pytest.mark.gpu


def _noalloc_run(m, n):
    dev = m.k.device
    cfg = m.cfg
    tok = torch.empty(n, cfg.batch, dtype=torch.int32, device=dev)
    lg = torch.empty(n, cfg.batch, cfg.vocab, dtype=torch.float32, device=dev)
    hd = torch.empty(n, cfg.batch, cfg.hidden, dtype=torch.float32, device=dev)
    workload.reset_state(m)
    io = _abi.xlpk_decode_io(0, lg.data_ptr(), hd.data_ptr(), 0, 0)
    st = get_lib().xlpk_decode_noalloc(m.engine.h, n, C.c_void_p(tok.data_ptr()), C.byref(io),
                                       C.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert st == _abi.XLPK_OK, get_lib().xlpk_last_cuda_error()
    m.engine.check()
    return tok.cpu(), lg.cpu(), hd.cpu()


def test_noalloc_matches_decode_on_two_calls(cuda_device):
    cfg = synth.get_config("tiny", steps=16)
    m = workload.build(cfg, device=cuda_device)
    ref = run_engine(m, cfg.steps)                       # xlpk_decode
    for _ in range(2):                                   # two calls in a row
        tok, lg, hd = _noalloc_run(m, cfg.steps)
        assert torch.equal(tok, ref.tokens)
        for s in range(cfg.steps):
            assert rel_l2(lg[s, 0], ref.logits[s, 0]) <= REL_L2_BF16
            assert rel_l2(hd[s, 0], ref.hidden[s, 0]) <= REL_L2_BF16
    # the handle's own decode still works after the no-alloc calls
    again = run_engine(m, cfg.steps)
    assert torch.equal(again.tokens, ref.tokens)


def test_noalloc_refuses_scratch_beyond_the_array(cuda_device):
    # 8 sequences x 8 kv heads x 148 CTAs of attention partials do not fit 8 MiB
    cfg = synth.get_config("tiny", hidden=512, n_q_heads=32, n_kv_heads=8, head_dim=128, ffn=512,
                           vocab=1024, kv_len=4, steps=2, batch=8)
    m = workload.build(cfg, device=cuda_device)
    tok = torch.empty(1, cfg.batch, dtype=torch.int32, device=cuda_device)
    workload.reset_state(m)
    with pytest.raises(XlpkError) as e:
        m.engine.decode_noalloc(1, tok)
    assert e.value.status == _abi.XLPK_ERR_UNSUPPORTED
    assert "static array" in str(e.value)
