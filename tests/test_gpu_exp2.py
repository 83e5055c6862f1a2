"""The FMA-pipe base-2 exponential used for part of the attention probabilities.

Its error must stay far below what bf16 probabilities can represent (8 significand bits,
relative step 3.9e-3): the bound checked here is 2e-4 relative against fp64 on the range the
softmax uses (x <= 8 after the lazy rescaling threshold), and exact zero below -125.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from block_sparse_attention_31_b200 import _lib
else:
    _lib = None


def test_exp2_polynomial_accuracy():
    g = torch.Generator("cpu").manual_seed(3)
    x = torch.cat([torch.linspace(-125.0, 8.0, 200001), torch.rand(100000, generator=g) * 133.0 - 125.0,
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, -124.999])]).float()
    xd = x.cuda()
    yp, ym = torch.empty_like(xd), torch.empty_like(xd)
    _lib.vsa_selftest_exp2(xd, yp, ym)
    torch.cuda.synchronize()
    ref = np.exp2(x.double().numpy())
    rel_poly = np.abs(yp.cpu().double().numpy() - ref) / ref
    rel_mufu = np.abs(ym.cpu().double().numpy() - ref) / ref
    assert rel_poly.max() < 2e-4, rel_poly.max()
    assert rel_mufu.max() < 2e-4


def test_exp2_polynomial_underflow_and_neg_inf():
    x = torch.tensor([-126.0, -200.0, -1e30, float("-inf")], device="cuda")
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    _lib.vsa_selftest_exp2(x, yp, ym)
    assert (yp.cpu() == 0).all()
    assert ym.cpu()[-1] == 0
