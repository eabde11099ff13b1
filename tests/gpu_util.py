"""Helpers shared by the GPU parity tests (test infrastructure)."""

import numpy as np
import torch

# Tolerances for bf16 outputs of the dense path (max abs, mean abs) and for the quantized
# path against the quantisation-emulating oracle (max abs).
DENSE_MAX_ABS = 1e-2
DENSE_MEAN_ABS = 1e-3
QUANT_MAX_ABS = 2e-2
# softmax statistics: fp32 accumulation of bf16 / int8 products and ex2.approx put the
# kernel within ~1e-5 relative of the fp64 oracle; these bounds leave two orders of margin.
STAT_MAX_RTOL = 1e-3
STAT_SUM_RTOL = 1e-3


def dev_bf16(bits: np.ndarray, device="cuda:0") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dev(x: np.ndarray, device="cuda:0") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def compare_out(got: np.ndarray, ref: np.ndarray, max_abs: float, mean_abs: float = None):
    """Compare where the oracle computed values (NaN = not sampled).  Returns (max, mean)."""
    sel = ~np.isnan(ref)
    assert sel.any()
    err = np.abs(got[sel] - ref[sel])
    assert np.all(np.isfinite(got[sel])), "non-finite output"
    mx, mn = float(err.max()), float(err.mean())
    assert mx <= max_abs, f"max abs error {mx:.3e} > {max_abs}"
    if mean_abs is not None:
        assert mn <= mean_abs, f"mean abs error {mn:.3e} > {mean_abs}"
    return mx, mn


def compare_stats(gmax: np.ndarray, gsum: np.ndarray, rmax: np.ndarray, rsum: np.ndarray):
    sel = ~np.isnan(rmax)
    gm, gs, rm, rs = gmax[sel], gsum[sel], rmax[sel], rsum[sel]
    dead = np.isneginf(rm)
    assert np.array_equal(np.isneginf(gm), dead), "fully masked rows differ"
    assert np.all(gs[dead] == 0)
    live = ~dead
    assert np.all(np.abs(gm[live] - rm[live]) <= STAT_MAX_RTOL * np.maximum(1.0, np.abs(rm[live])))
    assert np.all(np.abs(gs[live] - rs[live]) <= STAT_SUM_RTOL * np.abs(rs[live]))
