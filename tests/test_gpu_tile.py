"""The tcgen05 tensor-core tile of the batch-8 projections (xlpk_tc_gemm_tile)
against a float64 matrix product of the same operands, through the C ABI.

The weights and activations are bf16 values (the seeded generator's), so the
MMA's operands are exact and the only difference from the float64 product is
the fp32 accumulation; a second case feeds fp32 activations, which the tile
rounds to bf16 (round to nearest even) as they enter the MMA."""
import pytest
import torch

import synth
from persistent_decode_b200 import XlpkError, tc_gemm_tile

from tests.gpu_util import rel_l2

pytestmark = pytest.mark.gpu


def _operands(n, k, dev):
    w = synth.normal_bf16(11, f"tile.w.{n}x{k}", (n, k), 0.02, device="cpu")
    x = synth.normal_bf16(12, f"tile.x.{k}", (8, k), 1.0, device="cpu").float()
    return w, x


def _row_errors(y, ref):
    return ((y.double() - ref).abs().max(dim=1).values / ref.abs().max(dim=1).values.clamp_min(1e-30))


# one 128-row block with one K box; several blocks and boxes; a ragged last
# block with the largest K; a square case
@pytest.mark.parametrize("n,k", [(128, 64), (384, 256), (200, 4096), (1024, 1024)])
def test_tile_matches_float64_product(cuda_device, n, k):
    w, x = _operands(n, k, cuda_device)
    y = tc_gemm_tile(w.to(cuda_device), x.to(cuda_device)).cpu()
    ref = w.double() @ x.double().t()
    assert y.shape == (n, 8)
    assert rel_l2(y, ref) < 1e-5
    assert float(_row_errors(y, ref).max()) < 1e-4


def test_tile_rounds_fp32_activations_to_bf16(cuda_device):
    n, k = 256, 512
    w, xb = _operands(n, k, cuda_device)
    x = xb + synth.normal_fp32(13, "tile.dx", (8, k), 1e-3, device="cpu")
    y = tc_gemm_tile(w.to(cuda_device), x.to(cuda_device)).cpu()
    ref = w.double() @ x.to(torch.bfloat16).double().t()
    assert rel_l2(y, ref) < 1e-5


def test_tile_rejects_bad_shapes(cuda_device):
    w = torch.zeros(128, 96, dtype=torch.bfloat16, device=cuda_device)
    x = torch.zeros(8, 96, dtype=torch.float32, device=cuda_device)
    with pytest.raises(XlpkError):
        tc_gemm_tile(w, x)
