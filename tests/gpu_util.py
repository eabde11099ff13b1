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


# Quantized path only: a weight's FP16 and then E4M3 rounding is decided on 2^z computed by
# ex2.approx on the GPU and exactly in the oracle, so in rare rows one weight lands on the
# other side of an E4M3 rounding boundary.  softmax_sum is expressed against the row
# maximum (whose weight is ~1), so such a flip moves it by at most one E4M3 step of a weight
# <= 1, i.e. 1/8.  Those rows are allowed, up to this fraction of the rows.
E4M3_FLIP_ABS = 0.13
E4M3_FLIP_ROWS = 1e-3


def compare_stats(gmax: np.ndarray, gsum: np.ndarray, rmax: np.ndarray, rsum: np.ndarray, e4m3_flips: bool = False):
    sel = ~np.isnan(rmax)
    gm, gs, rm, rs = gmax[sel], gsum[sel], rmax[sel], rsum[sel]
    dead = np.isneginf(rm)
    assert np.array_equal(np.isneginf(gm), dead), "fully masked rows differ"
    assert np.all(gs[dead] == 0)
    live = ~dead
    assert np.all(np.abs(gm[live] - rm[live]) <= STAT_MAX_RTOL * np.maximum(1.0, np.abs(rm[live])))
    err = np.abs(gs[live] - rs[live])
    bad = err > STAT_SUM_RTOL * np.abs(rs[live])
    if not e4m3_flips:
        assert not bad.any(), f"{bad.sum()} rows: softmax_sum off by up to {err.max():.3e}"
        return
    n_bad, n_live = int(bad.sum()), int(live.sum())
    print(f"softmax_sum: {n_bad} of {n_live} rows beyond {STAT_SUM_RTOL} relative, max abs {err.max():.3e}")
    assert np.all(err <= E4M3_FLIP_ABS), f"softmax_sum off by {err.max():.3e} (more than one E4M3 step)"
    assert n_bad <= max(1, E4M3_FLIP_ROWS * n_live), f"{n_bad} of {n_live} rows beyond {STAT_SUM_RTOL}"
