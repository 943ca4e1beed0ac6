"""The V2 prefill's FMA-pipe 2^x (a quarter of its exponentials) against CUDA's exp2f on the
same device and against 2^x in float64.

The routine reduces x = n + f with n = rint(x), evaluates 2^f on [-0.5, 0.5] with a degree-4
polynomial fitted for minimax relative error (equioscillating at six points, 2.6e-6 in
exact arithmetic), adds n to the exponent and clamps x at -125 first. So on [-125, 0] its
relative error is the polynomial's plus fp32 rounding of the Horner steps (bound 3e-6), and
every x <= -125, -inf included (a masked key), gives the value at -125 (2^-125 to 1e-6).
"""
import numpy as np
import pytest
import torch

import differential_attention_05_b200 as da

pytestmark = pytest.mark.gpu

REL_BOUND = 3e-6


def _grid():
    # a dense grid over [-126, 0] (spacing 2^-12 plus a seeded jitter, so every fraction f
    # of the reduction is visited), the reduction's ties at +-0.5, and the clamp region
    rng = np.random.default_rng(2024)
    base = np.arange(-126 * 4096, 1, dtype=np.float64) / 4096.0
    jit = base + rng.uniform(-1.0 / 8192, 1.0 / 8192, base.size)
    ties = -np.arange(0, 126, dtype=np.float64) - 0.5
    x = np.concatenate([base, jit, ties, [0.0, -0.0, -125.0, -125.5, -126.0, -150.0, -1e30, -np.inf]])
    return np.clip(x, None, 0.0).astype(np.float32)


def test_exp2_fma2_against_exp2f_and_float64():
    x = _grid()
    y, y_ref = da.diffattn_selftest_exp2(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    y, y_ref = y.cpu().numpy().astype(np.float64), y_ref.cpu().numpy().astype(np.float64)
    inside = x >= -125.0
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y[inside] / exact[inside] - 1.0)
    rel_cuda = np.abs(y[inside] / y_ref[inside] - 1.0)
    assert rel.max() <= REL_BOUND, f"max rel err vs 2^x {rel.max():.3e}"
    assert rel_cuda.max() <= REL_BOUND + 2e-7, f"max rel err vs exp2f {rel_cuda.max():.3e}"
    # exp2f itself is within a couple of ulp of 2^x on this range (sanity of the comparison)
    assert np.max(np.abs(y_ref[inside] / exact[inside] - 1.0)) < 1e-6
    # the clamp: every x <= -125 (a masked key, -inf included) gives the value at -125,
    # 2^-125 to the polynomial's accuracy (its value at f = 0 is 1 - 7.2e-7)
    clamped = x <= -125.0
    assert np.all(y[clamped] == y[x == -125.0][0])
    assert abs(y[x == -125.0][0] / 2.0 ** -125 - 1.0) < 1e-6
    # integers are exact up to the polynomial's value at f = 0 (c0 = 1 - 7.2e-7)
    ints = (x == np.round(x)) & inside
    assert np.max(np.abs(y[ints] / exact[ints] - 1.0)) < 1e-6


def test_exp2_fma2_odd_length():
    # the routine works on pairs; an odd count leaves the last element alone
    x = torch.tensor([-1.0, -2.5, -0.25], dtype=torch.float32, device="cuda")
    y, y_ref = da.diffattn_selftest_exp2(x)
    torch.cuda.synchronize()
    np.testing.assert_allclose(y.cpu().numpy(), np.exp2(x.cpu().numpy()), rtol=3e-6)
