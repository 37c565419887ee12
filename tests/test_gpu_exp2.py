"""The kernels' exponentials against the mathematical 2^x (GPU).

The single-tile kernel computes one exponential pair in eight on the FMA pipe instead of the
MUFU: 2^x = 2^n * 2^f with n = rint(x) (rounding by adding and subtracting 1.5 * 2^23, the
round-to-nearest range reduction of Cody and Waite) and f = x - n in [-1/2, 1/2], 2^f from a
degree-3 polynomial fitted for least relative error on that interval, n added to the exponent
field.  Its stated accuracy: relative error below 7.7e-5 for x in [-125, 0], 0 for x < -125
(masked scores are -inf).  Checked on a dense grid, against fp64 2^x and against CUDA's own
exp2f (torch.exp2 on the device); the hardware ex2.approx path is checked the same way.
"""
import numpy as np
import pytest
import torch

import mixed_precision_tiled_b200 as mpt

pytestmark = pytest.mark.gpu

POLY_REL = 7.7e-5


def _grid():
    g = torch.Generator(device="cpu").manual_seed(5)
    dense = torch.linspace(-130.0, 0.0, 4_000_001, dtype=torch.float64)
    halves = torch.arange(-130, 1, dtype=torch.float64) + 0.5          # rounding ties
    ints = torch.arange(-130, 1, dtype=torch.float64)
    near = ints[:, None] + torch.tensor([-1e-6, 1e-6, -0.25, 0.25], dtype=torch.float64)
    rnd = -130.0 * torch.rand(1_000_000, generator=g, dtype=torch.float64)
    x = torch.cat([dense, halves, ints, near.reshape(-1), rnd]).float()
    return x[x <= 0]


def test_polynomial_exp2_error_bound():
    x = _grid().cuda()
    y = mpt.exp2_eval(x, 0)
    torch.cuda.synchronize()
    xd = x.double().cpu().numpy()
    yd = y.double().cpu().numpy()
    ref = np.exp2(xd)
    inside = xd >= -125.0
    rel = np.abs(yd[inside] - ref[inside]) / ref[inside]
    assert rel.max() < POLY_REL, rel.max()
    assert np.all(yd[~inside] == 0.0)
    # against CUDA's exp2f on the same inputs (its own error is far below the bound)
    cu = torch.exp2(x).double().cpu().numpy()
    rel_cu = np.abs(yd[inside] - cu[inside]) / cu[inside]
    assert rel_cu.max() < POLY_REL + 1e-6, rel_cu.max()
    assert np.all(np.isfinite(yd))


def test_hardware_exp2_path():
    x = _grid().cuda()
    y = mpt.exp2_eval(x, 1)
    torch.cuda.synchronize()
    xd = x.double().cpu().numpy()
    yd = y.double().cpu().numpy()
    normal = xd >= -126.0
    rel = np.abs(yd[normal] - np.exp2(xd[normal])) / np.exp2(xd[normal])
    assert rel.max() < 2.0 ** -20, rel.max()


def test_odd_length_and_masked_inputs():
    x = torch.tensor([0.0, -1.0, -0.5, float("-inf"), -200.0], device="cuda")
    y = mpt.exp2_eval(x, 0).cpu().numpy()
    assert np.allclose(y[:3], [1.0, 0.5, 2 ** -0.5], rtol=POLY_REL)
    assert y[3] == 0.0 and y[4] == 0.0
