"""Pins for the block-mask estimation oracle (block means, block scores, top-k)."""

import numpy as np
import pytest

from oracle import estimate
from workloads import bf16_bits_from_f32, bf16_bits_to_f32, iid_normal_bf16


def _bits(x):
    return bf16_bits_from_f32(np.asarray(x, dtype=np.float32))


def test_block_means_constant_and_affine():
    # x[r, d] = a_d + b_d * (r mod 64): integers of magnitude <= 130, exact in bf16, so each
    # block mean has a closed form (full blocks average r mod 64 over 0..63 twice -> 31.5;
    # the 44-row tail block 256..299 averages 0..43 -> 21.5)
    S, D = 300, 8
    r = (np.arange(S) % 64).astype(np.float32)[:, None]
    a = np.arange(D, dtype=np.float32)[None, :] - 3.0
    b = np.array([0, 1, -1, 2, 0, 1, 0, -2], dtype=np.float32)[None, :]
    x = (a + b * r)[None, None]
    got = estimate.block_means(_bits(x))
    assert got.shape == (1, 1, 3, D)
    for i, rmean in enumerate([31.5, 31.5, 21.5]):
        want = a[0].astype(np.float64) + b[0].astype(np.float64) * rmean
        assert np.array_equal(got[0, 0, i], want)
    c = estimate.block_means(_bits(np.full((2, 3, 200, 4), 1.5, np.float32)))
    assert np.all(c == 1.5)


def test_block_score_is_the_block_average_of_token_scores():
    # bilinearity: scale * mean(q) . mean(k) equals the mean over the block of scale * q_r . k_c
    B, Nq, Nkv, Sq, Skv, D, scale = 1, 4, 2, 300, 260, 16, 0.37
    q = iid_normal_bf16(31, 0, B, Nq, Sq, D)
    k = iid_normal_bf16(31, 1, B, Nkv, Skv, D)
    s = estimate.block_scores(estimate.block_means(q), estimate.block_means(k), scale)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    kf = bf16_bits_to_f32(k).astype(np.float64)
    for h in range(Nq):
        tok = scale * qf[0, h] @ kf[0, h // 2].T  # [Sq, Skv] token scores
        for i in range(3):
            for j in range(3):
                blk = tok[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
                assert abs(s[0, h, i, j] - blk.mean()) <= 1e-12 * max(1.0, abs(blk).max())


def _brute_topk(row, n):
    # repeated selection of the largest remaining score, first index on ties
    chosen, left = [], list(range(len(row)))
    for _ in range(n):
        best = left[0]
        for j in left[1:]:
            if row[j] > row[best]:
                best = j
        chosen.append(best)
        left.remove(best)
    out = np.zeros(len(row), np.uint8)
    out[chosen] = 1
    return out


@pytest.mark.parametrize("n_kb,n_keep", [(1, 1), (7, 3), (33, 10), (64, 64), (100, 1)])
def test_topk_matches_brute_force(n_kb, n_keep):
    rng = np.random.default_rng(n_kb * 100 + n_keep)
    scores = np.round(rng.standard_normal((5, n_kb)) * 4) / 4  # coarse values: many exact ties
    got = estimate.topk_mask(scores, n_keep)
    for r in range(5):
        assert np.array_equal(got[r], _brute_topk(scores[r], n_keep))
        assert got[r].sum() == n_keep


def test_topk_special_cases():
    s = np.array([[0.5, 2.0, 2.0, -1.0, 2.0]])
    assert np.array_equal(estimate.topk_mask(s, 1)[0], [0, 1, 0, 0, 0])   # argmax, first of the ties
    assert np.array_equal(estimate.topk_mask(s, 2)[0], [0, 1, 1, 0, 0])
    assert np.array_equal(estimate.topk_mask(s, 5)[0], [1, 1, 1, 1, 1])
    assert estimate.keep_count(512, 0.1) == 51 and estimate.keep_count(512, 0.5) == 256
    assert estimate.keep_count(3, 0.0) == 1 and estimate.keep_count(3, 1.0) == 3


def test_estimate_keeps_every_block_at_keep_one():
    q = iid_normal_bf16(32, 0, 1, 2, 400, 16)
    k = iid_normal_bf16(32, 1, 1, 1, 500, 16)
    m, s = estimate.estimate_block_mask(q, k, 0.25, 1.0)
    assert m.shape == (1, 2, 4, 4) and np.all(m == 1)
