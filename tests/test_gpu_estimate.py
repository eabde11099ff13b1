"""GPU parity of block-mask estimation (block means, pooled scores, top-k) against the oracle."""

import numpy as np
import pytest
import torch

import quantized_block_sparse_attn_b200 as qb
from oracle import estimate
from workloads import blocky_qk_bf16, iid_normal_bf16
from tests.gpu_util import dev, dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,N,S,D", [(1, 2, 300, 64), (2, 3, 1024, 128), (1, 1, 129, 256), (1, 4, 1, 128)])
def test_block_mean_parity(B, N, S, D):
    x = iid_normal_bf16(41, 0, B, N, S, D)
    got = qb.block_mean(dev_bf16(x)).cpu().numpy().astype(np.float64)
    want = estimate.block_means(x)
    # fp32 sums of at most 128 bf16 values of magnitude ~4: error below 128 * 2^-24 * 4 per mean
    assert np.abs(got - want).max() <= 4e-5


def _check_selection(mask, scores_ref, tol, n_keep):
    """Every row keeps n_keep blocks; rows whose cut is clear of the fp32 error match the oracle
    exactly; in every row each kept block scores at least every dropped block, up to tol."""
    m = mask.reshape(-1, mask.shape[-1]).astype(bool)
    s = scores_ref.reshape(-1, mask.shape[-1])
    t = tol.reshape(-1, mask.shape[-1])
    want = estimate.topk_mask(scores_ref, n_keep).reshape(m.shape).astype(bool)
    n_clear = 0
    for r in range(m.shape[0]):
        assert m[r].sum() == n_keep
        if n_keep < m.shape[1]:
            lo = s[r][m[r]].min()
            hi = s[r][~m[r]].max()
            assert lo >= hi - 2 * t[r].max(), f"row {r}: kept {lo} below dropped {hi}"
            order = np.sort(s[r])[::-1]
            if order[n_keep - 1] - order[n_keep] > 2 * t[r].max():
                n_clear += 1
                assert np.array_equal(m[r], want[r]), f"row {r} differs with a clear margin"
        else:
            assert m[r].all()
    return n_clear


@pytest.mark.parametrize("B,Nq,Nkv,nqb,nkb,D,keep", [
    (1, 4, 2, 5, 33, 128, 0.3), (2, 2, 1, 3, 512, 128, 0.1), (1, 1, 1, 2, 2048, 64, 0.5), (1, 2, 2, 1, 7, 128, 1.0),
])
def test_block_topk_parity(B, Nq, Nkv, nqb, nkb, D, keep):
    rng = np.random.default_rng(nkb + 17 * nqb)
    qm = rng.standard_normal((B, Nq, nqb, D)).astype(np.float32)
    km = rng.standard_normal((B, Nkv, nkb, D)).astype(np.float32)
    scale = D ** -0.5
    mask, sc = qb.block_topk(dev(qm), dev(km), scale, keep=keep, return_scores=True)
    qb.check()
    ref = estimate.block_scores(qm.astype(np.float64), km.astype(np.float64), scale)
    mag = scale * estimate.block_scores(np.abs(qm).astype(np.float64), np.abs(km).astype(np.float64), 1.0)
    tol = 1e-6 * mag
    assert np.all(np.abs(sc.cpu().numpy() - ref) <= tol)
    n_keep = estimate.keep_count(nkb, keep)
    _check_selection(mask.cpu().numpy(), ref, tol, n_keep)


def test_exact_ties_go_to_the_lower_block():
    # identical key blocks: all scores of a row tie, so the first n_keep blocks are kept
    qm = np.ones((1, 1, 2, 128), np.float32)
    km = np.ones((1, 1, 40, 128), np.float32)
    mask = qb.block_topk(dev(qm), dev(km), 0.5, n_keep=7).cpu().numpy()
    assert np.array_equal(mask[0, 0], np.tile((np.arange(40) < 7).astype(np.uint8), (2, 1)))


@pytest.mark.parametrize("S,keep", [(2048, 0.25), (4000, 0.1)])
def test_estimate_block_mask_on_blocky_inputs(S, keep):
    """The whole estimation on the structured Q/K recipe of the video workload (per-block means
    plus token noise), where block scores are well separated."""
    B, Nq, Nkv, D = 1, 4, 2, 128
    q = blocky_qk_bf16(42, "q", B, Nq, S, D)
    k = blocky_qk_bf16(42, "k", B, Nkv, S, D)
    scale = D ** -0.5
    mask, sc = qb.estimate_block_mask(dev_bf16(q), dev_bf16(k), scale, keep, return_scores=True)
    qb.check()
    want_mask, ref = estimate.estimate_block_mask(q, k, scale, keep)
    mag = scale * estimate.block_scores(np.abs(estimate.block_means(q)), np.abs(estimate.block_means(k)), 1.0)
    tol = 2e-5 * mag + 1e-6
    assert np.all(np.abs(sc.cpu().numpy() - ref) <= tol)
    n_clear = _check_selection(mask.cpu().numpy(), ref, tol, estimate.keep_count(ref.shape[-1], keep))
    assert n_clear >= 0.9 * Nq * ref.shape[2]  # the recipe separates blocks: nearly every row is exact
