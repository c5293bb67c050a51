"""The seeded input generators: published SplitMix64 outputs, rounding, distributions."""
import torch

import synth
from synth.gen import _GAMMA, _fp32_to_bf16_bits, _mix64, _mix64_int, _s64


def test_splitmix64_published_sequence():
    # SplitMix64 started from state 0 (Steele, Lea & Flood 2014; the reference
    # splitmix64.c) emits 0xe220a8397b1dcdaf, 0x6e789e6aa1b965f4, 0x06c45d188009454f.
    expect = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert [_mix64_int(i * _GAMMA) for i in (1, 2, 3)] == expect
    z = torch.tensor([_s64(i * _GAMMA) for i in (1, 2, 3)], dtype=torch.int64)
    got = [int(v) & ((1 << 64) - 1) for v in _mix64(z)]
    assert got == expect


def test_stream_is_counter_based():
    a = synth.splitmix64_stream(0, "w", 0, 1000)
    b = synth.splitmix64_stream(0, "w", 600, 400)
    assert torch.equal(a[600:], b)
    assert not torch.equal(a, synth.splitmix64_stream(1, "w", 0, 1000))
    assert not torch.equal(a, synth.splitmix64_stream(0, "w2", 0, 1000))


def test_bf16_rounding_matches_library():
    x = torch.randn(100000) * 0.02
    x = torch.cat([x, torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8])])
    ours = _fp32_to_bf16_bits(x).view(torch.bfloat16)
    assert torch.equal(ours.view(torch.int16), x.to(torch.bfloat16).view(torch.int16))


def test_normal_and_token_distributions():
    w = synth.normal_bf16(0, "dist", (512, 512), 0.02).float()
    assert abs(float(w.mean())) < 2e-4
    assert abs(float(w.std()) - 0.02) < 2e-4
    kurt = float(((w / w.std()) ** 4).mean())
    assert abs(kurt - 3.0) < 0.05                                      # Gaussian tails
    t = synth.uniform_tokens(5, "p", (200000,), 4096)
    assert int(t.min()) >= 0 and int(t.max()) < 4096
    counts = torch.bincount(t.long(), minlength=4096).float()
    assert 0.12 < float(counts.std() / counts.mean()) < 0.165          # Poisson: 1/sqrt(48.8)


def test_weight_shapes_and_fp8_layout():
    cfg = synth.get_config("tiny")
    w = synth.make_weights(cfg)
    assert w["layers.0.wq"].shape == (256, 256) and w["layers.1.w_down"].shape == (256, 1024)
    assert w["layers.0.wk"].shape == (128, 256) and w["embed"].dtype == torch.bfloat16
    fcfg = cfg.with_(weight_dtype="fp8_e4m3")
    wf = synth.make_weights(fcfg)
    assert wf["layers.0.w_gate"].dtype == torch.uint8
    assert wf["layers.0.w_gate.scale"].shape == (1024 // 128, 256 // 128)
    assert wf["embed"].dtype == torch.bfloat16
