"""Shared helpers of the GPU parity tests: tolerances and comparisons."""

from __future__ import annotations

import numpy as np
import torch

# bf16 inputs, bf16 P, fp32 accumulation and statistics, against the fp64 oracle
TOL_O = 2e-2
TOL_LSE = 5e-3
# attn_merge (and the fused accumulate epilogue) on identical fp32 partials, against
# the fp64 merge of the same partials: |dO| <= 1e-5 and |dLSE| <= 1e-5 + 2 ulp(|LSE|).
# The ulp term is the fp32 storage of the result: once |LSE| > 64 the spacing of fp32
# values (7.6e-6 at 64..128) is itself close to 1e-5, so rounding the exact LSE to
# fp32 can take up to half of it; two ulps leave room for the final add's rounding.
TOL_MERGE = 1e-5
MERGE_LSE_ULPS = 2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def ulp_fp32(x: np.ndarray) -> np.ndarray:
    """Spacing of fp32 numbers at |x| (the gap to the next fp32 value away from 0)."""
    a = np.abs(np.asarray(x, np.float64)).astype(np.float32)
    return (np.nextafter(a, np.float32(np.inf)) - a).astype(np.float64)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, tol_o=TOL_O, tol_lse=TOL_LSE, lse_ulps=0):
    """Element-wise check; -inf in LSE must match exactly. Each finite LSE may differ by
    tol_lse + lse_ulps * ulp_fp32(|LSE_ref|). Returns (max|dO|, max|dLSE|)."""
    o_gpu, lse_gpu = np.asarray(o_gpu, np.float64), np.asarray(lse_gpu, np.float64)
    o_ref, lse_ref = np.asarray(o_ref, np.float64), np.asarray(lse_ref, np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert lse_gpu.shape == lse_ref.shape, (lse_gpu.shape, lse_ref.shape)
    assert np.isfinite(o_gpu).all(), "non-finite O"
    ninf_g, ninf_r = np.isneginf(lse_gpu), np.isneginf(lse_ref)
    assert np.array_equal(ninf_g, ninf_r), f"-inf LSE pattern differs ({ninf_g.sum()} vs {ninf_r.sum()})"
    assert not np.isnan(lse_gpu).any(), "NaN LSE"
    do = float(np.abs(o_gpu - o_ref).max(initial=0.0))
    fin = ~ninf_r
    dl_abs = np.abs(lse_gpu[fin] - lse_ref[fin])
    bound = tol_lse + lse_ulps * ulp_fp32(lse_ref[fin])
    dl = float(dl_abs.max(initial=0.0))
    assert do <= tol_o, f"max|dO| = {do:.3e} > {tol_o}"
    if dl_abs.size:
        worst = int(np.argmax(dl_abs - bound))
        assert dl_abs[worst] <= bound[worst], (
            f"|dLSE| = {dl_abs[worst]:.3e} > {bound[worst]:.3e} at LSE {lse_ref[fin][worst]:.4f}")
    return do, dl
