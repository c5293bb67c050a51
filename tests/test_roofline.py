"""The roofline's algorithmic bytes per decode step, against parameter counts
worked out by hand for the two dense shapes (CPU only).

8B shape: 32 layers, hidden 4096, 32 q / 8 kv heads of 128, ffn 14336, vocab 128256.
  per layer: QKV (4096 + 2*1024) * 4096 + O 4096 * 4096 + FFN 3 * 14336 * 4096 = 218,103,808
  linear weights: 32 * 218,103,808 + LM head 128256 * 4096 = 7,504,658,432 elements (bf16)
  norm gains: 4 bytes * 4096 * (2 * 32 + 1) = 1,064,960
  K and V of one position, all layers: 32 * 8 * 128 * 2 values * 2 bytes = 131,072
1B shape: 16 layers, hidden 2048, 32 q / 8 kv heads of 64, ffn 8192, vocab 32000.
  per layer: (2048 + 2*512) * 2048 + 2048 * 2048 + 3 * 8192 * 2048 = 60,817,408
  linear weights: 16 * 60,817,408 + 32000 * 2048 = 1,038,614,528 elements
  norm gains: 4 * 2048 * 33 = 270,336; one position's K and V: 16 * 8 * 64 * 4 = 32,768
"""
import synth
from persistent_decode_b200 import roofline


def test_llama8b_step_bytes():
    cfg = synth.get_config("llama8b")
    w = 2 * 7_504_658_432 + 1_064_960
    assert roofline.weight_bytes(cfg) == w
    # new token at position 8192: 8193 positions read, one written, one embedding row (bf16)
    assert roofline.step_bytes(cfg, 8192) == w + 8193 * 131_072 + 131_072 + 4096 * 2


def test_llama1b_step_bytes():
    cfg = synth.get_config("llama1b")
    w = 2 * 1_038_614_528 + 270_336
    assert roofline.weight_bytes(cfg) == w
    assert roofline.step_bytes(cfg, 1024) == w + 1025 * 32_768 + 32_768 + 2048 * 2
    assert roofline.step_bytes(cfg, 1024, batch=4) == w + 4 * (1025 * 32_768 + 32_768 + 2048 * 2)


def test_fp8_counts_codes_and_block_scales():
    cfg = synth.get_config("llama8b_fp8")
    elems = 7_504_658_432
    assert roofline.weight_bytes(cfg) == elems + 4 * elems // (128 * 128) + 1_064_960


def test_call_bytes_sums_growing_steps():
    cfg = synth.get_config("tiny")
    assert roofline.call_bytes(cfg, 128, 3) == sum(roofline.step_bytes(cfg, 128 + s) for s in range(3))
    assert roofline.step_bytes(cfg, 129) - roofline.step_bytes(cfg, 128) == 2 * 2 * 64 * 2 * 2   # one more position


def test_moe_counts_only_active_experts():
    # 24 layers, hidden 2048, 16 q / 4 kv heads of 128, 64 experts (top-8) + 1 shared of width 1408, vocab 64000
    #   attention per layer: (2048 + 2*512) * 2048 + 2048 * 2048 = 10,485,760
    #   active experts per layer: (8 + 1) * 3 * 1408 * 2048 = 77,856,768
    #   linear elements: 24 * 88,342,528 + 64000 * 2048 = 2,251,292,672 (bf16)
    #   router (bf16, every layer): 64 * 2048 * 2 bytes = 262,144; norm gains 4 * 2048 * 49 = 401,408
    #   one position's K and V: 24 * 4 * 128 * 4 = 49,152
    cfg = synth.get_config("moe")
    w = 2 * 2_251_292_672 + 24 * 262_144 + 401_408
    assert roofline.weight_bytes(cfg) == w
    assert roofline.step_bytes(cfg, 4096) == w + 4097 * 49_152 + 49_152 + 2048 * 2
