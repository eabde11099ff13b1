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


# Quantized path against the plain reading of the oracle (weights E4M3(FP16(e^(s - m))) against
# the running max, moved at every block).  The kernel takes its weights against a power-of-two
# reference, so its E4M3 rounding falls on a shifted grid; the two readings differ by that
# rounding alone.  Every element is gated by the bound derived from E4M3's spacing
# (oracle.quant.qbsa_reading_gap_terms), plus the bf16 rounding of the output; the mean by
# PLAIN_MEAN_ABS (the readings' own mean distance is at most 3.7e-3 on the test inputs); and,
# where a caller asks for it (the Fig 4.1 workloads, whose rows keep thousands of keys), the
# maximum by QUANT_MAX_ABS.
PLAIN_MEAN_ABS = 1e-2


def check_qbsa(got, gmax, gsum, q8, k8, qs, ks, v8, vs, bm, scale, heads=None, q_blocks=None,
               plain_max_abs=None, e4m3_flips=False, tag=""):
    """Gate a qbsa_fwd result against both readings of the quantized oracle.  Returns the
    max abs errors (kernel's reading, plain reading)."""
    from oracle import quant
    args = (q8, k8, qs, ks, v8, vs, bm, scale)
    kw = dict(heads=heads, q_blocks=q_blocks)
    # tight: the kernel's own reading (lazy power-of-two reference)
    ref, rmax, rsum = quant.qbsa_forward_pow2ref(*args, **kw)
    e_pow2, _ = compare_out(got, ref, QUANT_MAX_ABS)
    compare_stats(gmax, gsum, rmax, rsum, e4m3_flips=e4m3_flips)
    # independent: the plain definition
    o_p, m_p, l_p = quant.qbsa_forward(*args, **kw)
    o_w, _, W = quant.qbsa_forward(*args, round_p=False, **kw)
    G, E = quant.qbsa_reading_gap_terms(*args, center=o_p, **kw)
    sel = ~np.isnan(m_p)
    live = sel & (l_p > 0)
    assert np.all(gsum[live] > 0)
    A = np.where(live, gsum, 1.0).astype(np.float64)
    gap = (G + W[..., None] * np.abs(o_w - o_p)) / A[..., None]
    bound = gap * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(o_p) + 1e-5
    err = np.abs(got - o_p)
    lv = np.broadcast_to(live[..., None], err.shape)
    bad = lv & ~(err <= bound)
    assert not bad.any(), f"{bad.sum()} elements beyond the derived bound vs the plain reading (max err {err[lv].max():.3e})"
    dead = sel & ~live
    assert np.all(got[dead] == 0)
    e_plain, mean_plain = float(err[lv].max()), float(err[lv].mean())
    assert mean_plain <= PLAIN_MEAN_ABS, f"mean abs error vs the plain reading {mean_plain:.3e}"
    if plain_max_abs is not None:
        assert e_plain <= plain_max_abs, f"max abs error vs the plain reading {e_plain:.3e} > {plain_max_abs}"
    assert np.all(np.abs(gmax[live] - m_p[live]) <= STAT_MAX_RTOL * np.maximum(1.0, np.abs(m_p[live])))
    assert np.all(np.abs(gsum[live] - l_p[live]) <= (E + np.abs(W - l_p))[live] * (1 + 1e-3) + 1e-5 * l_p[live])
    print(f"{tag} max abs err vs kernel's reading {e_pow2:.3e}; vs plain reading max {e_plain:.3e} "
          f"mean {mean_plain:.3e} (largest ratio to the derived bound {float((err[lv] / bound[lv]).max()):.3f})")
    return e_pow2, e_plain
