"""Pins of the quantisers and of the quantized block-sparse oracle."""

import numpy as np
import pytest

from oracle import formats, quant, dense
from workloads import bf16_bits_from_f32, bf16_bits_to_f32, block_keep_mask


def _bf16(rng, *shape, std=1.0):
    return bf16_bits_from_f32((std * rng.standard_normal(shape)).astype(np.float32))


def test_int8_quantiser_rounding_bound_and_extremes():
    rng = np.random.default_rng(1)
    x = _bf16(rng, 1, 2, 300, 16, std=3.0)
    codes, s = quant.quantize_qk_per_block(x)
    assert s.shape == (1, 2, 3)
    xf = bf16_to_f32 = bf16_bits_to_f32(x).astype(np.float64)
    for kb in range(3):
        r0, r1 = kb * 128, min(300, kb * 128 + 128)
        blk = xf[:, :, r0:r1]
        rec = codes[:, :, r0:r1].astype(np.float64) * s[:, :, kb, None, None]
        # |x - q s| <= s / 2, plus one float32 rounding of x / s (|x / s| <= 127: 127 * 2^-24)
        assert np.all(np.abs(blk - rec) <= s[:, :, kb, None, None] * (0.5 + 127 * 2.0 ** -24))
        # the block maximum maps to +-127, and s = amax / 127
        assert np.all(np.abs(codes[:, :, r0:r1]).max(axis=(2, 3)) == 127)
        assert np.allclose(s[:, :, kb], np.abs(blk).max(axis=(2, 3)) / 127, rtol=1e-7)
    assert bf16_to_f32 is not None


def test_int8_quantiser_zero_block():
    codes, s = quant.quantize_qk_per_block(np.zeros((1, 1, 128, 8), dtype=np.float32))
    assert np.all(codes == 0) and np.all(s == 1.0)


def test_e4m3_v_quantiser_bound_and_max_code():
    rng = np.random.default_rng(2)
    v = _bf16(rng, 1, 2, 500, 8, std=2.0)
    codes, s = quant.quantize_v_per_channel(v)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    rec = formats.e4m3_decode(codes) * s[:, :, None, :]
    # relative error <= 2^-4 (3 mantissa bits), plus the subnormal spacing 2^-10 * s
    assert np.all(np.abs(vf - rec) <= np.abs(vf) * 2.0 ** -4 + 2.0 ** -10 * s[:, :, None, :] * 1.0001)
    # the channel maximum lands on +-448
    amax_code = np.take_along_axis(codes, np.abs(vf).argmax(axis=2)[:, :, None, :], axis=2)
    assert np.all((amax_code & 0x7F) == 0x7E)


def _problem(seed, B=1, Nq=2, Nkv=1, Sq=300, Skv=270, D=16, keep=0.6):
    rng = np.random.default_rng(seed)
    q = _bf16(rng, B, Nq, Sq, D)
    k = _bf16(rng, B, Nkv, Skv, D)
    v = _bf16(rng, B, Nkv, Skv, D)
    q8, qs = quant.quantize_qk_per_block(q)
    k8, ks = quant.quantize_qk_per_block(k)
    v8, vs = quant.quantize_v_per_channel(v)
    nqb, nkb = -(-Sq // 128), -(-Skv // 128)
    bm = block_keep_mask(seed, B, Nq, nqb, nkb, keep)
    return dict(q=q, k=k, v=v, q8=q8, qs=qs, k8=k8, ks=ks, v8=v8, vs=vs, bm=bm)


def _direct_softmax(p, scale):
    """Plain (non-online) softmax over the kept keys of the dequantised problem, fp64."""
    q8, k8, v8 = p["q8"], p["k8"], p["v8"]
    B, Nq, Sq, D = q8.shape
    Nkv, Skv = k8.shape[1], k8.shape[2]
    out = np.zeros((B, Nq, Sq, D))
    for b in range(B):
        for h in range(Nq):
            g = h // (Nq // Nkv)
            t = q8[b, h].astype(np.int64) @ k8[b, g].astype(np.int64).T
            qsr = np.repeat(p["qs"][b, h], 128)[:Sq]
            ksr = np.repeat(p["ks"][b, g], 128)[:Skv]
            s = t * qsr[:, None].astype(np.float64) * ksr[None, :].astype(np.float64) * scale
            keep = np.repeat(np.repeat(p["bm"][b, h], 128, axis=0), 128, axis=1)[:Sq, :Skv].astype(bool)
            s = np.where(keep, s, -np.inf)
            w = np.exp(s - s.max(axis=1, keepdims=True))
            w /= w.sum(axis=1, keepdims=True)
            out[b, h] = (w @ formats.e4m3_decode(v8[b, g])) * p["vs"][b, g][None, :]
    return out


def test_online_recurrence_without_p_rounding_equals_direct_softmax():
    p = _problem(3)
    out, _, _ = quant.qbsa_forward(p["q8"], p["k8"], p["qs"], p["ks"], p["v8"], p["vs"], p["bm"], 0.25,
                                   round_p=False)
    assert np.allclose(out, _direct_softmax(p, 0.25), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("seed,D,scale", [(10, 16, 0.5), (11, 64, 0.2), (12, 128, 128 ** -0.5)])
def test_power_of_two_reference_matches_final_max_up_to_subnormals(seed, D, scale):
    """The lazily moved power-of-two reference gives the codes of the order-free
    definition p8 = E4M3(2^(z - ceil(max z))) except where a weight falls in E4M3's
    subnormal range (below 2^-6) on one side: each such weight moves by at most the
    subnormal spacing 2^-9 (in units of the final reference), which bounds the output."""
    from oracle.formats import e4m3_decode, e4m3_encode
    p = _problem(seed, Nq=1, Nkv=1, Sq=128, Skv=1024, D=D, keep=1.0)
    got, _, _ = quant.qbsa_forward(p["q8"], p["k8"], p["qs"], p["ks"], p["v8"], p["vs"], p["bm"], scale)
    q8, k8 = p["q8"][0, 0].astype(np.int64), p["k8"][0, 0].astype(np.int64)
    ks_col = np.repeat(p["ks"][0, 0].astype(np.float64), 128)
    z = (q8 @ k8.T) * (float(p["qs"][0, 0, 0]) * ks_col[None, :] * scale) / np.log(2.0)
    M = np.ceil(z.max(axis=1))
    w = np.exp2(z - M[:, None])
    w8 = e4m3_decode(e4m3_encode(w.astype(np.float16).astype(np.float32)))
    vdq = e4m3_decode(p["v8"][0, 0]) * p["vs"][0, 0][None, :]
    two_pass = (w8 @ vdq) / w8.sum(axis=1)[:, None]
    n_sub = (w < 2.0 ** -6).sum(axis=1)
    bound = 2 * n_sub * 2.0 ** -9 * np.abs(vdq).max() / w8.sum(axis=1)
    assert np.all(np.abs(got[0, 0] - two_pass) <= bound[:, None] + 1e-12)


def test_loops_equal_vectorised_tiny():
    p = _problem(4, Nq=2, Nkv=1, Sq=140, Skv=200, D=4, keep=1.0)
    a = quant.qbsa_forward(p["q8"], p["k8"], p["qs"], p["ks"], p["v8"], p["vs"], p["bm"], 0.5)
    b = quant.qbsa_forward_loops(p["q8"], p["k8"], p["qs"], p["ks"], p["v8"], p["vs"], p["bm"], 0.5)
    for x, y in zip(a, b):
        assert np.allclose(x, y, rtol=1e-12, atol=1e-12)


def test_zero_query_gives_exact_counts_and_mean():
    p = _problem(5)
    q8 = np.zeros_like(p["q8"])
    out, mx, sm = quant.qbsa_forward(q8, p["k8"], p["qs"], p["ks"], p["v8"], p["vs"], p["bm"], 0.25)
    Skv = p["k8"].shape[2]
    vdq = formats.e4m3_decode(p["v8"][0, 0]) * p["vs"][0, 0][None, :]
    for h in range(2):
        for qb in range(p["bm"].shape[2]):
            kept = np.nonzero(p["bm"][0, h, qb])[0]
            cols = np.concatenate([np.arange(kb * 128, min(Skv, kb * 128 + 128)) for kb in kept])
            r0, r1 = qb * 128, min(300, qb * 128 + 128)
            assert np.all(sm[0, h, r0:r1] == len(cols))  # p8 = 1 exactly
            assert np.all(mx[0, h, r0:r1] == 0.0)
            assert np.allclose(out[0, h, r0:r1], vdq[cols].mean(axis=0)[None, :], rtol=1e-13, atol=1e-13)


def test_constant_v_returns_v_exactly():
    p = _problem(6)
    v8 = np.full_like(p["v8"], 0x3B)            # 1.375 in every entry
    out, _, _ = quant.qbsa_forward(p["q8"], p["k8"], p["qs"], p["ks"], v8, p["vs"], p["bm"], 0.25)
    want = 1.375 * p["vs"][0, 0].astype(np.float64)
    assert np.allclose(out[0], np.broadcast_to(want, out[0].shape), rtol=1e-14, atol=0)


def test_unkept_blocks_have_no_influence():
    p = _problem(7, keep=0.5)
    a = quant.qbsa_forward(p["q8"], p["k8"], p["qs"], p["ks"], p["v8"], p["vs"], p["bm"], 0.25)
    k8, v8 = p["k8"].copy(), p["v8"].copy()
    # blocks not kept by ANY query block of head 0 and 1 may be overwritten freely
    unused = np.nonzero(p["bm"][0].max(axis=(0, 1)) == 0)[0]
    assert len(unused) >= 0
    for kb in unused:
        k8[:, :, kb * 128:(kb + 1) * 128] = 99
        v8[:, :, kb * 128:(kb + 1) * 128] = 0x70
    b = quant.qbsa_forward(p["q8"], k8, p["qs"], p["ks"], v8, p["vs"], p["bm"], 0.25)
    for x, y in zip(a, b):
        assert np.array_equal(x, y, equal_nan=True)


def test_unkept_rows_are_zero():
    p = _problem(8)
    bm = p["bm"].copy()
    bm[0, 1, 1, :] = 0
    out, mx, sm = quant.qbsa_forward(p["q8"], p["k8"], p["qs"], p["ks"], p["v8"], p["vs"], bm, 0.25)
    assert np.all(out[0, 1, 128:256] == 0) and np.all(mx[0, 1, 128:256] == -np.inf) and np.all(sm[0, 1, 128:256] == 0)


def test_all_blocks_kept_tracks_unquantised_attention():
    # quantisation error is small on N(0,1) data: loose sanity pin (the article gives no figure)
    p = _problem(9, Sq=256, Skv=256, D=64, keep=1.0)
    out, _, _ = quant.qbsa_forward(p["q8"], p["k8"], p["qs"], p["ks"], p["v8"], p["vs"], p["bm"], 64 ** -0.5)
    ref, _, _ = dense.attention_forward(p["q"], p["k"], p["v"][:, [0, 0]], layout="BNSD", scale=64 ** -0.5)
    err = np.abs(out - ref)
    assert err.max() < 0.05 and err.mean() < 0.01


@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_block_mask_generator_counts_and_diagonal(keep):
    bm = block_keep_mask(3, 1, 4, 16, 16, keep)
    n = max(1, int(round(keep * 16)))
    assert np.all(bm.sum(axis=3) == n)
    assert np.all(bm[0, :, np.arange(16), np.arange(16)] == 1)
