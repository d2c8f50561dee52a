"""Shared helpers of the GPU parity tests: tolerances and comparisons."""

from __future__ import annotations

import numpy as np
import torch

# bf16 inputs, bf16 P, fp32 accumulation and statistics, against the fp64 oracle
TOL_O = 2e-2
TOL_LSE = 5e-3
# attn_merge on identical fp32 partials against the fp64 merge of the same partials.
# LSE is stored in fp32, whose spacing exceeds 1e-5 once |LSE| > 64, so that bound is
# applied relative to max(1, |LSE|).
TOL_MERGE = 1e-5


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def compare(o_gpu, lse_gpu, o_ref, lse_ref, tol_o=TOL_O, tol_lse=TOL_LSE, rel_lse=False):
    """Element-wise check; -inf in LSE must match exactly. Returns (max|dO|, max|dLSE|)."""
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
    if rel_lse:
        dl_abs = dl_abs / np.maximum(1.0, np.abs(lse_ref[fin]))
    dl = float(dl_abs.max(initial=0.0))
    assert do <= tol_o, f"max|dO| = {do:.3e} > {tol_o}"
    assert dl <= tol_lse, f"max|dLSE| = {dl:.3e} > {tol_lse}"
    return do, dl
