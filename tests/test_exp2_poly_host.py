"""Host-side checks of the FMA-pipe 2^x that the softmax uses for part of its
exponentials (sm100_ptx.cuh, exp2_poly_f32x2), without a GPU.

1. The constants in the kernel source are the fp32 rounding of the minimax fit that
   csrc/exp2_poly_fit.py produces (Remez exchange on [-1/2, 1/2], relative error).
2. The method as the kernel runs it - x clamped at -126, Cody and Waite's reduction
   x = n + f with n = round(x) through the 1.5 * 2^23 shifter, the degree-3 polynomial
   by Horner's rule with one rounding per fused multiply-add, and n added to the
   result's exponent field as an integer - emulated in fp32 with numpy, stays within
   the fit's bound (7.48e-5) plus a few fp32 roundings of 2^x for x >= -125.5, and
   gives tiny non-negative values below that.
"""

from __future__ import annotations

import importlib.util
import re
from pathlib import Path

import numpy as np

CSRC = Path(__file__).resolve().parents[1] / "online_softmax_exact_b200" / "csrc"
POLY_REL = 7.48e-5 + 4 * 2.0 ** -24


def _kernel_constants() -> dict[str, np.float32]:
    src = (CSRC / "sm100_ptx.cuh").read_text()
    out = {}
    for name in ("kExp2Shift", "kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3"):
        m = re.search(rf"constexpr float {name} = ([0-9.eE+-]+)f;", src)
        assert m, name
        out[name] = np.float32(float(m.group(1)))
    return out


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", CSRC / "exp2_poly_fit.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fma32(a, b, c):
    """fp32 fused multiply-add: the product of two fp32 values is exact in fp64, so one
    rounding of the fp64 sum to fp32 is the fused operation's (up to the rare double
    rounding of the fp64 sum, far below the bound checked here)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _poly_exp2(x: np.ndarray, k: dict[str, np.float32]) -> np.ndarray:
    x = x.astype(np.float32)
    xc = np.maximum(x, np.float32(-126.0))
    sh = k["kExp2Shift"]
    t = (xc + sh).astype(np.float32)                      # n in the low mantissa bits
    f = (xc - (t - sh).astype(np.float32)).astype(np.float32)
    p = _fma32(f, np.full_like(f, k["kExp2C3"]), np.full_like(f, k["kExp2C2"]))
    p = _fma32(p, f, np.full_like(f, k["kExp2C1"]))
    p = _fma32(p, f, np.full_like(f, k["kExp2C0"]))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_kernel_constants_are_the_rounded_fit():
    k = _kernel_constants()
    assert k["kExp2Shift"] == np.float32(1.5 * 2.0 ** 23)
    c32, err = _fit_module().remez_exp2(3)
    for i in range(4):
        assert k[f"kExp2C{i}"] == c32[i], (i, k[f"kExp2C{i}"], c32[i])
    assert err <= 7.48e-5


def test_emulated_method_within_its_bound():
    k = _kernel_constants()
    rng = np.random.default_rng(11)
    grid = np.linspace(-125.5, 127.0, 1_000_001)
    ints = np.arange(-125, 127, dtype=np.float64)
    edges = np.concatenate([ints, ints + 0.5, ints - 0.5])
    x = np.concatenate([grid, rng.uniform(-125.5, 127.0, 500_000), edges]).astype(np.float32)
    x = x[x >= np.float32(-125.5)]
    # neighbours of the rounding boundaries of the reduction
    x = np.concatenate([x, np.nextafter(x, np.float32(200)), np.nextafter(x, np.float32(-200))])
    x = x[(x >= np.float32(-125.5)) & (x < np.float32(127.0))]
    y = _poly_exp2(x, k).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y / exact - 1.0)
    assert np.all(np.isfinite(y))
    assert float(rel.max()) <= POLY_REL, float(rel.max())


def test_emulated_method_below_the_clamp():
    k = _kernel_constants()
    x = np.array([-126.0, -127.0, -300.0, -1e30], dtype=np.float32)
    y = _poly_exp2(x, k).astype(np.float64)
    assert np.all(y >= 0.0) and np.all(y <= 2.0 ** -125)


def test_a_wrong_coefficient_breaks_the_bound():
    """The check has teeth: one coefficient off by 1e-3 exceeds the bound."""
    k = dict(_kernel_constants())
    k["kExp2C2"] = np.float32(k["kExp2C2"] * np.float32(1.001))
    x = np.linspace(-4.0, 4.0, 100_001).astype(np.float32)
    rel = np.abs(_poly_exp2(x, k).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert float(rel.max()) > POLY_REL
