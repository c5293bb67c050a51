"""Engine vs oracle, element by element, through the C ABI on a B200."""
import pytest
import torch

import synth
from persistent_decode_b200 import workload

from tests.gpu_util import compare_with_oracle, oracle_for, rel_l2, run_engine

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny(cuda_device):
    return workload.build(synth.get_config("tiny"), device=cuda_device)


def test_generator_device_matches_host(cuda_device):
    w_gpu = synth.normal_bf16(0, "layers.0.wq", (256, 256), 0.02, device=cuda_device).cpu()
    w_cpu = synth.normal_bf16(0, "layers.0.wq", (256, 256), 0.02, device="cpu")
    assert torch.equal(w_gpu.view(torch.int16), w_cpu.view(torch.int16))
    t_gpu = synth.uniform_tokens(1, "prompt", (1000,), 32000, device=cuda_device).cpu()
    assert torch.equal(t_gpu, synth.uniform_tokens(1, "prompt", (1000,), 32000))


def test_tiny_prefill_cache_matches_oracle(tiny):
    o = oracle_for(tiny)
    T = tiny.cfg.kv_len
    k_gpu = tiny.k[:, :, :, :T].float().cpu()
    v_gpu = tiny.v[:, :, :, :T].float().cpu()
    assert rel_l2(k_gpu, o.K[:, :, :, :T].float()) < 1e-2
    assert rel_l2(v_gpu, o.V[:, :, :, :T].float()) < 1e-2
    # positions beyond the prompt were never written
    assert int(tiny.k[:, :, :, T:].abs().sum().item()) == 0


@pytest.mark.parametrize("unfused", [False, True], ids=["persistent", "kernel_per_op"])
def test_tiny_decode_matches_oracle(tiny, unfused):
    run = run_engine(tiny, tiny.cfg.steps, unfused=unfused)
    o = oracle_for(tiny)
    compare_with_oracle(tiny, run, o, tiny.cfg.steps)


def test_tiny_persistent_matches_kernel_per_op(tiny):
    # the same tiles and arithmetic in the same order (the fused FFN's split-K
    # partial sums meet in a fixed-point accumulator, whose integer adds do not
    # depend on arrival order): bit-identical results
    a = run_engine(tiny, tiny.cfg.steps, unfused=False)
    b = run_engine(tiny, tiny.cfg.steps, unfused=True)
    assert torch.equal(a.tokens, b.tokens)
    assert torch.equal(a.logits, b.logits)
    assert torch.equal(a.hidden, b.hidden)


def test_tiny_runs_are_bit_identical(tiny):
    runs = [run_engine(tiny, tiny.cfg.steps) for _ in range(3)]
    for r in runs[1:]:
        assert torch.equal(r.logits, runs[0].logits)
        assert torch.equal(r.hidden, runs[0].hidden)


def test_debug_logits_hold_the_last_step(tiny):
    # parity mode: buffers registered once, overwritten by every step
    from persistent_decode_b200 import XlpkError
    cfg, dev = tiny.cfg, tiny.k.device
    ref = run_engine(tiny, 6)
    lg = torch.full((cfg.batch, cfg.vocab), float("nan"), dtype=torch.float32, device=dev)
    hd = torch.full((cfg.batch, cfg.hidden), float("nan"), dtype=torch.float32, device=dev)
    tiny.engine.debug_logits(lg, hd)
    try:
        workload.reset_state(tiny)
        tok = torch.empty(6, cfg.batch, dtype=torch.int32, device=dev)
        tiny.engine.decode(6, tok)
        tiny.engine.check()
        assert torch.equal(lg.cpu(), ref.logits[5])
        assert torch.equal(hd.cpu(), ref.hidden[5])
    finally:
        tiny.engine.debug_logits(None, None)
    with pytest.raises(XlpkError):
        tiny.engine.debug_logits(lg.view(-1)[1:], None)   # 4 bytes in: not 16-byte aligned


def test_fused_ffn_matches_two_stage_ffn(cuda_device):
    # gate/up + split-K down in one stage (default for bf16 dense models) vs
    # gate/up and down as two stages (XLPK_FLAG_NO_FUSED_FFN), same weights
    from persistent_decode_b200 import _abi
    cfg = synth.get_config("tiny", steps=10)
    fused = workload.build(cfg, device=cuda_device, norm_std=0.1)
    two = workload.build(cfg, device=cuda_device, norm_std=0.1, weights=fused.weights,
                         flags=_abi.XLPK_FLAG_NO_FUSED_FFN)
    assert two.engine.info().kernels_per_step_unfused == 5 * cfg.n_layers + 1
    assert fused.engine.info().kernels_per_step_unfused == 4 * cfg.n_layers + 1
    a = run_engine(fused, cfg.steps)
    b = run_engine(two, cfg.steps)
    assert torch.equal(a.tokens, b.tokens)
    assert rel_l2(a.logits, b.logits) < 1e-5
    compare_with_oracle(two, b, oracle_for(two), cfg.steps)


def test_tiny_decode_is_deterministic_and_resumable(tiny):
    a = run_engine(tiny, 16)
    # the same 16 steps as two calls of 8 (state carried in the handle)
    workload.reset_state(tiny)
    dev = tiny.k.device
    t1 = torch.empty(8, 1, dtype=torch.int32, device=dev)
    t2 = torch.empty(8, 1, dtype=torch.int32, device=dev)
    tiny.engine.decode(8, t1)
    tiny.engine.decode(8, t2)
    tiny.engine.check()
    assert torch.equal(torch.cat([t1, t2]).cpu(), a.tokens)


def test_kernel_per_op_graph_replay_matches_eager(tiny):
    # the kernel-per-op launches recorded by stream capture into a CUDA graph
    # (each call clears its dependency counters on the stream) and replayed
    cfg, dev = tiny.cfg, tiny.k.device
    n = 6
    a = run_engine(tiny, n, unfused=True)
    workload.reset_state(tiny)
    tok = torch.full((n, cfg.batch), -1, dtype=torch.int32, device=dev)
    lg = torch.zeros(n, cfg.batch, cfg.vocab, dtype=torch.float32, device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        tiny.engine.decode(n, tok, logits=lg, unfused=True)
    g.replay()
    torch.cuda.synchronize()
    tiny.engine.check()
    assert torch.equal(tok.cpu(), a.tokens)
    assert rel_l2(lg.cpu(), a.logits) < 1e-5
    del g


def test_decode_resumes_across_launch_modes(tiny):
    # 8 kernel-per-op steps, then 8 persistent steps on the same handle, equal
    # 16 persistent steps: the persistent call continues from the counters the
    # kernel-per-op call left
    a = run_engine(tiny, 16)
    workload.reset_state(tiny)
    dev = tiny.k.device
    t1 = torch.empty(8, 1, dtype=torch.int32, device=dev)
    t2 = torch.empty(8, 1, dtype=torch.int32, device=dev)
    tiny.engine.decode(8, t1, unfused=True)
    tiny.engine.decode(8, t2)
    tiny.engine.check()
    assert torch.equal(torch.cat([t1, t2]).cpu(), a.tokens)


def test_tiny_kv_append_positions_exact(tiny):
    cfg = tiny.cfg
    T, n = cfg.kv_len, cfg.steps
    before = tiny.k[:, :, :, :T].clone()
    run = run_engine(tiny, n)
    # the prompt's entries are untouched, each step wrote exactly its position
    assert torch.equal(tiny.k[:, :, :, :T], before)
    written = tiny.k[:, :, :, T:T + n].float().abs().sum(dim=-1)
    assert bool((written > 0).all())
    o = oracle_for(tiny)
    compare_with_oracle(tiny, run, o, n)
    assert rel_l2(tiny.k[:, :, :, T:T + n].float().cpu(), o.K[:, :, :, T:T + n].float()) < 1e-2
    assert rel_l2(tiny.v[:, :, :, T:T + n].float().cpu(), o.V[:, :, :, T:T + n].float()) < 1e-2


@pytest.mark.parametrize("batch", [2, 4])
def test_tiny_batched_with_gains(cuda_device, batch):
    cfg = synth.get_config("tiny", batch=batch, steps=12)
    m = workload.build(cfg, device=cuda_device, norm_std=0.1)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps)


def test_cache_tail_garbage_is_ignored(cuda_device):
    # positions at and beyond the current length are not part of the sequence:
    # fill them with NaN (what an uninitialised cache may hold) and the decode
    # must be unaffected, since each step writes its position before reading it
    cfg = synth.get_config("tiny", steps=10)
    m = workload.build(cfg, device=cuda_device)
    T = cfg.kv_len
    m.k[:, :, :, T:] = float("nan")
    m.v[:, :, :, T:] = float("nan")
    run = run_engine(m, cfg.steps)
    assert bool(torch.isfinite(run.hidden).all())
    compare_with_oracle(m, run, oracle_for(m), cfg.steps)


def test_tiny_ragged_grid(cuda_device):
    # a grid size that divides nothing evenly: every stage gets ragged CTA spans
    cfg = synth.get_config("tiny", steps=6)
    m = workload.build(cfg, device=cuda_device, n_ctas=37)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps)


def test_generate_with_host_buffers(tiny):
    ref = run_engine(tiny, 8)
    out = torch.empty(8, 1, dtype=torch.int32).pin_memory()
    tiny.engine.generate(tiny.start_tokens.tolist(), [tiny.cfg.kv_len], 8, out)
    assert torch.equal(out, ref.tokens)


def test_kv_full_is_rejected(tiny):
    from persistent_decode_b200 import XlpkError
    workload.reset_state(tiny)
    tok = torch.empty(tiny.cfg.steps + 1, 1, dtype=torch.int32, device=tiny.k.device)
    with pytest.raises(XlpkError) as e:
        tiny.engine.decode(tiny.cfg.steps + 1, tok)
    assert e.value.status == -5


def test_weights_may_be_freed_after_create(tiny, cuda_device):
    """The engine keeps its own copies (packed weights, embedding, norm gains)."""
    from persistent_decode_b200 import Engine
    ref = run_engine(tiny, 8)
    w2 = {k: v.clone() for k, v in tiny.weights.items()}
    k2, v2 = tiny.k.clone(), tiny.v.clone()
    eng = Engine(tiny.cfg, w2, k2, v2)
    del w2
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    junk = torch.full((64 << 20,), 7, dtype=torch.int32, device=cuda_device)   # reuse the freed memory
    eng.set_state(tiny.start_tokens.tolist(), [tiny.cfg.kv_len])
    tok = torch.empty(8, 1, dtype=torch.int32, device=cuda_device)
    eng.decode(8, tok)
    eng.check()
    assert torch.equal(tok.cpu(), ref.tokens)
    del junk
    eng.close()


def test_head_dim_128_group_4_multi_chunk(cuda_device):
    # d = 128 and 4 query heads per kv head (the 8B/MoE attention shape) at a
    # size the oracle finishes quickly; KV 200 spans several 64-position chunks
    # with a ragged tail, and n_ctas 148 leaves CTAs without attention work.
    cfg = synth.get_config("tiny", hidden=512, n_q_heads=4, n_kv_heads=1, head_dim=128,
                           ffn=1024, kv_len=200, steps=10)
    m = workload.build(cfg, device=cuda_device, norm_std=0.1)
    for unfused in (False, True):
        run = run_engine(m, cfg.steps, unfused=unfused)
        compare_with_oracle(m, run, oracle_for(m), cfg.steps)


def test_llama1b_full_size_prefix(cuda_device):
    # the 1B shape at its full size (KV 1024 from a 1024-token prompt prefilled
    # through the engine, the whole grid): the oracle replays the first steps.
    cfg = synth.get_config("llama1b")
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, 24)
    o = oracle_for(m)
    T = cfg.kv_len
    assert rel_l2(m.k[:, :, :, :T].float().cpu(), o.K[:, :, :, :T].float()) < 1e-2
    compare_with_oracle(m, run, o, 3)
    assert int(run.tokens.min()) >= 0 and int(run.tokens.max()) < cfg.vocab


def test_llama8b_full_size_prefix(cuda_device):
    # the 8B shape with its 8192-entry synthetic cache, in the launch
    # configuration the bench times (one CTA per SM, one launch per call)
    cfg = synth.get_config("llama8b")
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, 16)
    o = oracle_for(m)
    compare_with_oracle(m, run, o, 2)
    T = cfg.kv_len
    # steps wrote exactly positions T .. T+15
    assert bool((m.k[:, :, :, T:T + 16].float().abs().sum(-1) > 0).all())
    assert int(m.k[:, :, :, T + 16:].float().abs().sum().item()) == 0


def test_llama1b_batch4_prefix(cuda_device):
    # the 1B shape at batch 4 (four independent prompts), with a 64-token
    # prompt per sequence so that the oracle's prefill stays short; the
    # activation region holds 4 x 8192 floats, so the ring keeps 2 slots
    cfg = synth.get_config("llama1b", batch=4, kv_len=64, steps=8)
    m = workload.build(cfg, device=cuda_device)
    assert m.engine.info().ring_slots >= 2
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), 3)
    T = cfg.kv_len
    # every sequence wrote exactly positions T .. T+7 of its own cache rows
    assert bool((m.k[:, :, :, T:T + 8].float().abs().sum(-1) > 0).all())
    assert int(m.k[:, :, :, T + 8:].float().abs().sum().item()) == 0


@pytest.mark.parametrize("batch", [2, 4])
def test_windowed_down_projection_matches_whole_k(cuda_device, batch):
    # the down projection streamed in K windows of 1024 columns (4 windows of
    # F = 4096) against the same model with the whole K staged at once: the
    # per-lane sums run over the same chunks in the same order
    from persistent_decode_b200 import _abi
    cfg = synth.get_config("tiny", ffn=4096, batch=batch, steps=6)
    two = _abi.XLPK_FLAG_NO_FUSED_FFN
    whole = workload.build(cfg, device=cuda_device, norm_std=0.1, flags=two)
    win = workload.build(cfg, device=cuda_device, norm_std=0.1, weights=whole.weights, flags=two, window=1024)
    for unfused in (False, True):
        a = run_engine(whole, cfg.steps, unfused=unfused)
        b = run_engine(win, cfg.steps, unfused=unfused)
        assert torch.equal(a.tokens, b.tokens)
        assert torch.equal(a.logits, b.logits)
    compare_with_oracle(win, b, oracle_for(win), cfg.steps)


@pytest.mark.parametrize("unfused", [False, True], ids=["persistent", "kernel_per_op"])
def test_batch8_tensor_core_path_matches_oracle(cuda_device, unfused):
    # batch 8 runs every projection on tcgen05 MMAs (bf16 activations as the B
    # operand, fp32 accumulators in tensor memory)
    cfg = synth.get_config("tiny", batch=8, steps=6)
    m = workload.build(cfg, device=cuda_device, norm_std=0.1)
    run = run_engine(m, cfg.steps, unfused=unfused)
    compare_with_oracle(m, run, oracle_for(m), cfg.steps)


def test_batch8_tensor_core_windowed_down_matches_whole_k(cuda_device):
    # the tensor-core down projection over K windows of 1024 columns keeps
    # accumulating in the same tensor-memory columns, in the same K order, as
    # the whole K staged at once (window 4096 = F): identical results
    cfg = synth.get_config("tiny", ffn=4096, batch=8, steps=4)
    whole = workload.build(cfg, device=cuda_device, norm_std=0.1, window=4096)
    win = workload.build(cfg, device=cuda_device, norm_std=0.1, weights=whole.weights, window=1024)
    a = run_engine(whole, cfg.steps)
    b = run_engine(win, cfg.steps)
    assert torch.equal(a.tokens, b.tokens)
    assert torch.equal(a.logits, b.logits)
    compare_with_oracle(win, b, oracle_for(win), cfg.steps)


def test_batch8_tensor_cores_match_cuda_cores(cuda_device):
    # the MMA's B operand carries each input as a bf16 high part and a bf16
    # remainder (about 16 significant bits), so the tensor-core decode agrees
    # with the fp32 CUDA-core tiles to ~1e-4, far inside the 1e-2 tolerance
    from persistent_decode_b200 import _abi
    cfg = synth.get_config("tiny", batch=8, steps=6)
    tc = workload.build(cfg, device=cuda_device, norm_std=0.1)
    cc = workload.build(cfg, device=cuda_device, norm_std=0.1, weights=tc.weights,
                        flags=_abi.XLPK_FLAG_NO_TENSOR_CORES)
    a = run_engine(tc, cfg.steps)
    b = run_engine(cc, cfg.steps)
    assert torch.equal(a.tokens, b.tokens)
    assert rel_l2(a.logits, b.logits) < 1e-3
    assert rel_l2(a.hidden, b.hidden) < 1e-3
    compare_with_oracle(cc, b, oracle_for(cc), cfg.steps)


def test_llama1b_batch8_tensor_core_prefix(cuda_device):
    cfg = synth.get_config("llama1b", batch=8, kv_len=32, steps=4)
    m = workload.build(cfg, device=cuda_device)
    run = run_engine(m, cfg.steps)
    compare_with_oracle(m, run, oracle_for(m), 2)
