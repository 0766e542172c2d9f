"""The FMA-pipe exponential on the device (msa_debug_exp2_fma, the helper the dense teacher-LSE loop
uses for part of its exponentials) against float64 2^x: relative error <= 3e-7 on [-125, 1/2], and
2^-125 (tiny, positive) below that range and at -inf."""
import pytest
import torch

import block_sparse_attention_idx_b200 as msa

pytestmark = pytest.mark.gpu


def test_exp2_fma_relative_error_on_its_range():
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.linspace(-125.0, 0.5, 1 << 20, dtype=torch.float64),
                   -125.0 + 125.5 * torch.rand(1 << 18, generator=g, dtype=torch.float64),
                   torch.tensor([0.0, -0.5, 0.5, -1.0, -2.0, -1e-30, -124.5, -125.0], dtype=torch.float64)])
    x = x.to(torch.float32)
    y = msa.msa_debug_exp2_fma(x.cuda()).cpu().double()
    ref = torch.exp2(x.double())
    rel = ((y - ref) / ref).abs().max().item()
    print(f"exp2_fma max relative error {rel:.3e} over {x.numel()} values")
    assert rel <= 3e-7


def test_exp2_fma_below_range_and_odd_length():
    x = torch.tensor([-float("inf"), -1000.0, -126.0, -125.5, 0.25], dtype=torch.float32)  # odd count
    y = msa.msa_debug_exp2_fma(x.cuda()).cpu().double()
    assert torch.all(y[:4] > 0) and torch.all(y[:4] <= 2.0 ** -124)
    assert abs(y[4].item() / 2.0 ** 0.25 - 1) <= 3e-7
