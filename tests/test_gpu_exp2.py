"""The polynomial 2^x of the attention softmax against CUDA's exp2f.

Part of the softmax's exponentials run on the FMA pipe: Cody-Waite range
reduction x = n + f (n = round(x), f in [-0.5, 0.5]), 2^f by a cubic fitted in
this project by the Remez exchange on relative error, 2^n added to the
exponent field.  The fit's bound is 7.5e-5 relative error over [-125, 0]
(below -125 the argument is raised to -125, keeping 2^n a normal number); the
bf16 probabilities it feeds are rounded to 2^-9 relative.
"""
import numpy as np
import pytest
import torch

import step_adaptive_sparse_b200 as area

pytestmark = pytest.mark.gpu


def _poly(x: torch.Tensor) -> torch.Tensor:
    y = torch.empty_like(x)
    area.area_test_exp2_poly(x, y, x.numel())
    torch.cuda.synchronize()
    return y


def test_exp2_poly_relative_error_bound():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 0.0, 1 << 20), -rng.random(1 << 18) * 30.0,
                        np.arange(-125, 1, dtype=np.float64),            # integers
                        np.arange(-125, 0) + 0.5]).astype(np.float32)   # half-way points
    dx = torch.from_numpy(x).cuda()
    got = _poly(dx).double()
    want = torch.exp2(dx).double()                   # CUDA's exp2f
    rel = ((got - want).abs() / want).max().item()
    assert rel < 8e-5, rel
    assert torch.all(got > 0)


def test_exp2_poly_below_the_range_and_masked_keys():
    x = torch.tensor([-125.0, -126.0, -1000.0, -float("inf"), 0.0, -1e-30],
                     dtype=torch.float32, device="cuda")
    got = _poly(x).cpu().double().numpy()
    floor = 2.0 ** -125
    assert abs(got[0] - floor) <= 1e-4 * floor
    for v in got[1:4]:                               # clamped to 2^-125
        assert abs(v - floor) <= 1e-4 * floor
    assert abs(got[4] - 1.0) < 8e-5 and abs(got[5] - 1.0) < 8e-5


def test_exp2_poly_odd_length():
    x = torch.linspace(-10, 0, 1001, device="cuda")
    got = _poly(x).double()
    want = torch.exp2(x).double()
    assert ((got - want).abs() / want).max().item() < 8e-5
