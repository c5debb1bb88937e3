"""The epilogues' activation functions against their definitions in fp64.

GELU(x) = x Phi(x) with Phi the standard normal CDF (the ViT3 MLP inner model's GELU;
erf-based, not the tanh approximation) and GELU'(x) = Phi(x) + x phi(x); SiLU(x) = x sigma(x)
(the SwiGLU / GLU gate) and SiLU'(x) = sigma(x) (1 + x (1 - sigma(x))).  The device GELU takes
erf from Abramowitz & Stegun 7.1.26 (|error| <= 1.5e-7) with hardware reciprocal and
exponential approximations; the SiLU's sigma uses the hardware tanh approximation.  The fused
apply evaluates GELU alone with erf from Abramowitz & Stegun 7.1.28 (|error| <= 3e-7, one
reciprocal).  All must stay far below the bf16 rounding (2^-9 relative) that every output of
theirs gets.
"""
import math

import pytest
import torch

pytestmark = pytest.mark.gpu


def _exact(kind, x):
    x = x.double()
    if kind == "gelu":
        cdf = 0.5 * (1.0 + torch.special.erf(x / math.sqrt(2.0)))
        pdf = torch.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
        return x * cdf, cdf + x * pdf
    s = torch.sigmoid(x)
    return x * s, s * (1.0 + x * (1.0 - s))


@pytest.mark.parametrize("kind,tol", [("gelu", 1e-6), ("silu", 2e-3)])
def test_activation_against_its_definition(kind, tol):
    from weight_sequence_mixing_b200 import binding

    x = torch.cat([torch.linspace(-12.0, 12.0, 200001), torch.randn(100000) * 3.0,
                   torch.tensor([0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0, 1e4, -1e4])]).float().cuda()
    y, dy = binding.selftest_activation(kind, x)
    torch.cuda.synchronize()
    ey, edy = _exact(kind, x.cpu())
    # absolute error relative to the size of the value (|x| + 1): GELU(x) ~ x for large x
    scale = x.cpu().double().abs() + 1.0
    err_y = ((y.cpu().double() - ey).abs() / scale).max().item()
    err_dy = ((dy.cpu().double() - edy).abs()).max().item()
    assert err_y <= tol, f"{kind}: {err_y:.3e}"
    assert err_dy <= tol, f"{kind}': {err_dy:.3e}"
    assert torch.isfinite(y).all() and torch.isfinite(dy).all()


def test_apply_gelu_against_its_definition():
    from weight_sequence_mixing_b200 import binding

    x = torch.cat([torch.linspace(-12.0, 12.0, 200001), torch.randn(100000) * 3.0,
                   torch.tensor([0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0, 1e4, -1e4])]).float().cuda()
    y, dy = binding.selftest_activation("gelu_fwd", x)
    torch.cuda.synchronize()
    ey, _ = _exact("gelu", x.cpu())
    scale = x.cpu().double().abs() + 1.0
    err = ((y.cpu().double() - ey).abs() / scale).max().item()
    assert err <= 1e-6, f"apply GELU: {err:.3e}"
    assert torch.isfinite(y).all() and (dy == 0).all()
