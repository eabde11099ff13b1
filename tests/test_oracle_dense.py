"""Pins of the dense oracle against what the definition and mathematics fix.

Each pin is chosen so that a plausible slip in the oracle fails one of them: a
missing scale, pse scaled or dropped, the mask polarity flipped, a causal vertex
placed at the wrong corner, a transposed operand, a wrong GQA head map, a wrong
TND offset, or stats taken from the wrong max.
"""

import numpy as np
import pytest
import torch

from oracle import dense
from oracle.dense import INF_TOKENS


def _rand(rng, *shape):
    return rng.standard_normal(shape)


CASES = [
    dict(sq=7, skv=7, mode=0, pre=INF_TOKENS, nxt=INF_TOKENS),
    dict(sq=9, skv=13, mode=0, pre=2, nxt=3),
    dict(sq=9, skv=13, mode=0, pre=0, nxt=0),
    dict(sq=11, skv=6, mode=0, pre=-2, nxt=4),
    dict(sq=8, skv=8, mode=2, pre=INF_TOKENS, nxt=INF_TOKENS),
    dict(sq=10, skv=7, mode=2, pre=INF_TOKENS, nxt=INF_TOKENS),
    dict(sq=6, skv=11, mode=3, pre=INF_TOKENS, nxt=INF_TOKENS),
    dict(sq=11, skv=6, mode=3, pre=INF_TOKENS, nxt=INF_TOKENS),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("with_pse", [False, True])
def test_vectorised_equals_loops(case, with_pse):
    rng = np.random.default_rng(11)
    d = 5
    q, k, v = _rand(rng, case["sq"], d), _rand(rng, case["skv"], d), _rand(rng, case["skv"], 4)
    ok = dense.allowed(case["sq"], case["skv"], case["mode"], case["pre"], case["nxt"])
    pse = _rand(rng, case["sq"], case["skv"]) if with_pse else None
    a = dense.attend(q, k, v, 0.37, ok, pse)
    b = dense.attend_loops(q, k, v, 0.37, ok, pse)
    for x, y in zip(a, b):
        assert np.allclose(x, y, rtol=1e-12, atol=1e-12, equal_nan=True)


def test_mask_polarity_and_modes_by_hand():
    # atten_mask: 1 = masked (guide §4.2)
    am = np.array([[0, 1, 0], [1, 1, 0], [0, 0, 0]], dtype=np.uint8)
    ok = dense.allowed(3, 3, 0, INF_TOKENS, INF_TOKENS, am)
    assert ok.tolist() == [[True, False, True], [False, False, True], [True, True, True]]
    # mode 2: top-left vertex; mode 3: bottom-right vertex (guide §4.3)
    assert dense.allowed(2, 4, 2).tolist() == [[True, False, False, False], [True, True, False, False]]
    assert dense.allowed(2, 4, 3).tolist() == [[True, True, True, False], [True, True, True, True]]
    # band: i - pre <= j <= i + next
    assert dense.allowed(3, 5, 0, 1, 1).tolist() == [
        [True, True, False, False, False], [True, True, True, False, False], [False, True, True, True, False]]


def test_matches_torch_sdpa_unmasked_and_causal():
    rng = np.random.default_rng(3)
    q, k, v = _rand(rng, 1, 3, 37, 16), _rand(rng, 1, 3, 37, 16), _rand(rng, 1, 3, 37, 16)
    for mode, causal in ((0, False), (2, True)):
        out, _, _ = dense.attention_forward(q, k, v, layout="BNSD", scale=0.21, sparse_mode=mode)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=causal, scale=0.21)
        assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_matches_torch_sdpa_boolean_mask_mode3_and_pse():
    rng = np.random.default_rng(4)
    sq, skv = 9, 21
    q, k, v = _rand(rng, 1, 2, sq, 8), _rand(rng, 1, 2, skv, 8), _rand(rng, 1, 2, skv, 8)
    pse = _rand(rng, 1, 2, sq, skv)
    out, _, _ = dense.attention_forward(q, k, v, layout="BNSD", scale=0.5, sparse_mode=3, pse=pse)
    keep = torch.from_numpy(dense.allowed(sq, skv, 3))
    bias = torch.from_numpy(pse).masked_fill(~keep, float("-inf"))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=bias, scale=0.5)
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", [0, 2, 3])
def test_zero_query_gives_uniform_weights_and_integer_counts(mode):
    rng = np.random.default_rng(5)
    sq, skv = 12, 9
    q = np.zeros((1, 1, sq, 4))
    k, v = _rand(rng, 1, 1, skv, 4), _rand(rng, 1, 1, skv, 3)
    out, mx, sm = dense.attention_forward(q, k, v, layout="BNSD", scale=1.0, sparse_mode=mode,
                                          pre_tokens=2, next_tokens=1)
    ok = dense.allowed(sq, skv, mode, 2, 1)
    for i in range(sq):
        cnt = ok[i].sum()
        assert sm[0, 0, i] == cnt  # exact integer
        if cnt:
            assert mx[0, 0, i] == 0.0
            assert np.allclose(out[0, 0, i], v[0, 0][ok[i]].mean(axis=0), rtol=1e-13, atol=1e-13)
        else:
            assert mx[0, 0, i] == -np.inf and np.all(out[0, 0, i] == 0.0)


def test_constant_v_returns_v_and_single_key_rows():
    rng = np.random.default_rng(6)
    q, k = _rand(rng, 1, 2, 10, 6), _rand(rng, 1, 2, 10, 6)
    v = np.broadcast_to(np.array([1.5, -2.25, 3.0]), (1, 2, 10, 3)).copy()
    out, _, sm = dense.attention_forward(q, k, v, layout="BNSD", scale=0.3, sparse_mode=2)
    assert np.allclose(out, v, rtol=1e-14, atol=1e-14)
    v2 = _rand(rng, 1, 2, 10, 3)
    out2, mx2, sm2 = dense.attention_forward(q, k, v2, layout="BNSD", scale=0.3, sparse_mode=2)
    # causal row 0 sees only key 0: O = V_0, sum = 1, max = the single score
    assert np.allclose(out2[0, :, 0], v2[0, :, 0], rtol=0, atol=1e-15)
    assert np.all(sm2[0, :, 0] == 1.0)
    assert np.allclose(mx2[0, :, 0], 0.3 * np.einsum("hd,hd->h", q[0, :, 0], k[0, :, 0]), rtol=1e-14)


def test_stats_reproduce_logsumexp():
    # softmax_max + log(softmax_sum) is the log-sum-exp of the masked scores
    from scipy.special import logsumexp
    rng = np.random.default_rng(8)
    q, k, v = _rand(rng, 1, 1, 17, 8), _rand(rng, 1, 1, 23, 8), _rand(rng, 1, 1, 23, 8)
    _, mx, sm = dense.attention_forward(q, k, v, layout="BNSD", scale=0.7, sparse_mode=3)
    s = 0.7 * q[0, 0] @ k[0, 0].T
    s[~dense.allowed(17, 23, 3)] = -np.inf
    assert np.allclose(mx[0, 0] + np.log(sm[0, 0]), logsumexp(s, axis=1), rtol=1e-13)
    assert np.allclose(mx[0, 0], s.max(axis=1), rtol=1e-14, atol=0)


def test_mode3_equals_mode2_when_square_and_band_defaults_are_unmasked():
    rng = np.random.default_rng(9)
    q, k, v = _rand(rng, 1, 2, 13, 4), _rand(rng, 1, 2, 13, 4), _rand(rng, 1, 2, 13, 4)
    a = dense.attention_forward(q, k, v, layout="BNSD", scale=0.4, sparse_mode=2)
    b = dense.attention_forward(q, k, v, layout="BNSD", scale=0.4, sparse_mode=3)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    band0 = dense.attention_forward(q, k, v, layout="BNSD", scale=0.4, sparse_mode=0, pre_tokens=0, next_tokens=0)
    assert np.allclose(band0[0], v, rtol=0, atol=1e-15)  # only the diagonal key


def test_bsnd_is_transposed_bnsd():
    rng = np.random.default_rng(10)
    q, k, v = _rand(rng, 2, 3, 11, 4), _rand(rng, 2, 3, 14, 4), _rand(rng, 2, 3, 14, 4)
    a = dense.attention_forward(q, k, v, layout="BNSD", scale=0.3, sparse_mode=3)
    t = lambda x: np.ascontiguousarray(np.swapaxes(x, 1, 2))  # noqa: E731
    b = dense.attention_forward(t(q), t(k), t(v), layout="BSND", scale=0.3, sparse_mode=3)
    assert np.allclose(t(a[0]), b[0], rtol=0, atol=0)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


def test_gqa_equals_repeated_kv_heads():
    rng = np.random.default_rng(12)
    q = _rand(rng, 1, 6, 9, 4)
    k, v = _rand(rng, 1, 2, 9, 4), _rand(rng, 1, 2, 9, 4)
    a = dense.attention_forward(q, k, v, layout="BNSD", scale=0.5, sparse_mode=3)
    kr, vr = np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1)  # heads 0,1,2 -> kv 0; 3,4,5 -> kv 1
    b = dense.attention_forward(q, kr, vr, layout="BNSD", scale=0.5, sparse_mode=3)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_tnd_equals_per_sequence_bnsd():
    rng = np.random.default_rng(13)
    lens_q, lens_k = [5, 9, 3], [7, 9, 6]
    cq, ck = np.cumsum(lens_q), np.cumsum(lens_k)
    q = _rand(rng, cq[-1], 4, 8)
    k, v = _rand(rng, ck[-1], 2, 8), _rand(rng, ck[-1], 2, 8)
    out, mx, sm = dense.attention_forward(q, k, v, layout="TND", scale=0.35, sparse_mode=3,
                                          actual_seq_qlen=cq, actual_seq_kvlen=ck)
    for b in range(3):
        q0, q1 = (cq[b - 1] if b else 0), cq[b]
        k0, k1 = (ck[b - 1] if b else 0), ck[b]
        qb = np.swapaxes(q[q0:q1], 0, 1)[None]
        kb, vb = np.swapaxes(k[k0:k1], 0, 1)[None], np.swapaxes(v[k0:k1], 0, 1)[None]
        o2, m2, s2 = dense.attention_forward(qb, kb, vb, layout="BNSD", scale=0.35, sparse_mode=3)
        assert np.allclose(np.swapaxes(out[q0:q1], 0, 1), o2[0], rtol=0, atol=1e-15)
        assert np.array_equal(mx[:, q0:q1], m2[0]) and np.array_equal(sm[:, q0:q1], s2[0])


def test_pse_row_shift_moves_max_only():
    rng = np.random.default_rng(14)
    q, k, v = _rand(rng, 1, 1, 8, 4), _rand(rng, 1, 1, 10, 4), _rand(rng, 1, 1, 10, 4)
    pse = _rand(rng, 1, 1, 8, 10)
    shift = rng.standard_normal(8)
    a = dense.attention_forward(q, k, v, layout="BNSD", scale=0.6, pse=pse)
    b = dense.attention_forward(q, k, v, layout="BNSD", scale=0.6, pse=pse + shift[None, None, :, None])
    assert np.allclose(a[0], b[0], rtol=1e-13, atol=1e-13)
    assert np.allclose(b[1] - a[1], shift[None, None], rtol=1e-13, atol=1e-13)
    assert np.allclose(a[2], b[2], rtol=1e-13)


def test_bf16_bits_input_equals_float_input():
    from workloads import bf16_bits_from_f32, bf16_bits_to_f32
    rng = np.random.default_rng(15)
    qb = bf16_bits_from_f32(rng.standard_normal((1, 1, 6, 4)).astype(np.float32))
    kb = bf16_bits_from_f32(rng.standard_normal((1, 1, 6, 4)).astype(np.float32))
    a = dense.attention_forward(qb, kb, kb, layout="BNSD", scale=0.5)
    b = dense.attention_forward(bf16_bits_to_f32(qb), bf16_bits_to_f32(kb), bf16_bits_to_f32(kb),
                                layout="BNSD", scale=0.5)
    assert np.array_equal(a[0], b[0])


def test_tile_sets_by_hand():
    # no mask, skv = 300: three k-tiles, only the tail tile is partial
    ts = dense.tile_sets(200, 300, 0)
    assert ts == [([0, 1, 2], [2]), ([0, 1, 2], [2])]
    # top-left causal, 256 x 256: tile 0 sees {0} (partial); tile 1 sees {0, 1}, 1 partial
    assert dense.tile_sets(256, 256, 2) == [([0], [0]), ([0, 1], [1])]
    # bottom-right causal with skv = sq + 128 shifts the diagonal one tile right
    assert dense.tile_sets(256, 384, 3) == [([0, 1], [1]), ([0, 1, 2], [2])]
