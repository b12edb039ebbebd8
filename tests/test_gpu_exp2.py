"""GPU: the fused kernel's FMA-pipe 2^x against fp64 exp2 and its derived error bound."""
import math

import pytest
import torch

from sequence_exact_attention_ring_b200 import binding

pytestmark = pytest.mark.gpu

BOUND = 1.02e-4  # exp2_poly.h: max relative error of the fp32 polynomial on [-1/2, 1/2]


def run(x):
    x = x.contiguous().cuda()
    y = torch.empty_like(x)
    rc = binding.ring_attn_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    return y.cpu()


def test_relative_error_within_bound(cuda_lib):
    x = torch.linspace(-126.0, 8.0, 2_000_000, dtype=torch.float32)
    y = run(x).double()
    ref = torch.exp2(x.double())
    rel = ((y - ref) / ref).abs().max().item()
    assert rel <= BOUND, rel
    # the same inputs through CUDA's own exp2 stay within a few ulp: the bound is the polynomial's
    cu = torch.exp2(x.cuda()).cpu().double()
    assert ((cu - ref) / ref).abs().max().item() < 1e-6


def test_special_values(cuda_lib):
    x = torch.tensor([-math.inf, -1000.0, -127.0, 0.0, 1.0, 8.0, -0.5, 0.5], dtype=torch.float32)
    y = run(x)
    assert y[0].item() == 0.0 and y[1].item() == 0.0 and y[2].item() == 0.0
    assert y[3].item() == 1.0 and y[4].item() == 2.0 and y[5].item() == 256.0
    assert abs(y[6].item() / 2 ** -0.5 - 1) <= BOUND and abs(y[7].item() / 2 ** 0.5 - 1) <= BOUND


def test_large_arguments_saturate_at_2_pow_127(cuda_lib):
    """Above 127 the exponent field would wrap; the polynomial clamps, so a row sum of its
    results shows the overflow instead of hiding it."""
    x = torch.tensor([127.0, 128.0, 200.0, 1000.0, math.inf, 126.0], dtype=torch.float32)
    y = run(x)
    for v in y[:5].tolist():
        assert v == 2.0 ** 127
    assert y[5].item() == 2.0 ** 126
