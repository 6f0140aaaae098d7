"""The softmax's FMA-pipe exponential against CUDA's exp2 and its stated error bound."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_exp2_poly_error_bound(gpu_lib):
    # softmax arguments are s*c - m <= 8 (the running maximum may lag by up to 2^8)
    x = torch.cat([torch.linspace(-125.0, 8.0, 2_000_001, device="cuda"),
                   -torch.rand(1_000_000, device="cuda") * 30.0,
                   torch.tensor([0.0, -0.5, -1.0, -1e-7, -20.0, -124.9, 7.99, 8.0],
                                device="cuda")])
    y = torch.empty_like(x)
    gpu_lib.lf_debug_exp2_poly(x, y)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 1e-4, rel
    # CUDA's own fp32 exp2 for comparison: both are within the bound of the reference
    assert ((torch.exp2(x).double() - ref).abs() / ref).max().item() < 1e-6
    # masked logits (-inf) and deep underflow give (almost) zero
    z = torch.tensor([-float("inf"), -127.0, -200.0, -1e30], device="cuda")
    yz = torch.empty_like(z)
    gpu_lib.lf_debug_exp2_poly(z, yz)
    assert (yz >= 0).all() and (yz < 1.3e-38).all() and torch.isfinite(yz).all()
