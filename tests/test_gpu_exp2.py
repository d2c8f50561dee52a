"""The FMA-pipe 2^x the softmax uses for part of its exponentials, against the exact
value and against the exp unit's ex2.approx (the other path of the same softmax).

Method (the kernel's own): Cody and Waite's reduction x = n + f with n = round(x),
|f| <= 1/2, a degree-3 polynomial for 2^f fitted by the Remez exchange algorithm for
minimax relative error (csrc/exp2_poly_fit.py: 7.48e-5 after rounding the coefficients
to fp32), and n added to the exponent field. Bound checked here: relative error <=
7.48e-5 plus a few fp32 roundings (2^-22) against 2^x in fp64 for x >= -125.5. Just
above -126 (n = -126) the polynomial's value below 1 makes the result denormal: the
error there is checked in absolute terms (<= 2^-138). Inputs below -126 give a value in
[0, 2^-125].
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

POLY_REL = 7.48e-5 + 4 * 2.0 ** -24


@pytest.fixture(scope="module")
def osx():
    import online_softmax_exact_b200 as m

    return m


def _xs():
    g = torch.Generator().manual_seed(5)
    grid = torch.linspace(-126.0, 127.0, 2_000_001, dtype=torch.float64)
    rnd = torch.rand(1_000_000, generator=g, dtype=torch.float64) * 253.0 - 126.0
    # integers, half-integers and their neighbours: the reduction's rounding boundaries
    ints = torch.arange(-126, 128, dtype=torch.float64)
    edges = torch.cat([ints, ints + 0.5, ints - 0.5]).clamp(-126, 127)
    x = torch.cat([grid, rnd, edges]).to(torch.float32)
    x = torch.cat([x, torch.nextafter(x, torch.full_like(x, 200.0)),
                   torch.nextafter(x, torch.full_like(x, -200.0))]).clamp(-126, 127)
    return x


def test_poly_within_its_bound_of_the_exact_value(osx):
    x = _xs()
    y = osx.attn_debug_exp2(x.cuda(), use_poly=True).cpu().double()
    exact = torch.exp2(x.double())
    assert torch.isfinite(y).all()
    normal = x >= -125.5
    rel = ((y[normal] - exact[normal]) / exact[normal]).abs()
    worst = float(rel.max())
    print(f"polynomial 2^x: max relative error {worst:.3e} (bound {POLY_REL:.3e})")
    assert worst <= POLY_REL
    # n = -126: the result may be denormal, absolutely tiny errors only
    assert float((y[~normal] - exact[~normal]).abs().max()) <= 2.0 ** -138


def test_poly_against_the_exp_unit(osx):
    """Both exponentials of the softmax agree to the polynomial's bound plus the exp
    unit's own error (2^-22 relative for ex2.approx.ftz at normal results)."""
    x = _xs()
    x = x[x >= -125.0]              # keep ex2.approx's results normal (no flush to zero)
    xg = x.cuda()
    yp = osx.attn_debug_exp2(xg, use_poly=True).cpu().double()
    ye = osx.attn_debug_exp2(xg, use_poly=False).cpu().double()
    rel = ((yp - ye) / ye).abs()
    worst = float(rel.max())
    print(f"polynomial vs ex2.approx: max relative difference {worst:.3e}")
    assert worst <= POLY_REL + 2.0 ** -21


def test_poly_below_the_clamp_and_special_points(osx):
    x = torch.tensor([-126.0, -127.0, -300.0, -1e30, 0.0, 1.0, -1.0, 0.5, -0.5, 100.0],
                     dtype=torch.float32)
    y = osx.attn_debug_exp2(x.cuda(), use_poly=True).cpu().double().numpy()
    assert np.all(y[:4] >= 0.0) and np.all(y[:4] <= 2.0 ** -125)
    exact = np.exp2(x[4:].double().numpy())
    assert np.all(np.abs(y[4:] / exact - 1.0) <= POLY_REL)
    # odd length: the last value is handled on its own
    y1 = osx.attn_debug_exp2(torch.tensor([3.0], device="cuda"), use_poly=True).cpu()
    assert abs(float(y1[0]) / 8.0 - 1.0) <= POLY_REL
