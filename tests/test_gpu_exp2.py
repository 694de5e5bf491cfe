"""The polynomial exponential used inside the attention kernel against the
float64 exponential: relative error <= 1e-4 on [-100, 8] (well inside the
bf16 rounding of the probabilities, 2^-9); below that the result is a
finite, non-negative value under 2^-99."""

import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_polynomial_exp2_relative_error(ress_gpu):
    x = torch.cat([torch.linspace(-100.0, 8.0, 2_000_001), torch.tensor([0.0, -0.5, 0.5, 7.99])])
    x = x.to(torch.float32).cuda()
    y = torch.empty_like(x)
    st = ress_gpu.lib.ress_test_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                     x.numel(), None)
    assert st == 0
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel <= 1e-4, rel
    tail = torch.tensor([-100.5, -120.0, -125.9, -126.0, -127.0, -1000.0, -1e30], device="cuda")
    yt = torch.empty_like(tail)
    assert ress_gpu.lib.ress_test_exp2(ctypes.c_void_p(tail.data_ptr()),
                                       ctypes.c_void_p(yt.data_ptr()), tail.numel(), None) == 0
    torch.cuda.synchronize()
    assert torch.isfinite(yt).all() and (yt >= 0).all() and (yt < 2.0 ** -99).all()
