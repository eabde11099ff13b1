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


READINGS = {"plain": quant.qbsa_forward, "pow2ref": quant.qbsa_forward_pow2ref}
LOOPS = {"plain": quant.qbsa_forward_loops, "pow2ref": quant.qbsa_forward_pow2ref_loops}


def _args(p, scale, **over):
    d = dict(q8=p["q8"], k8=p["k8"], qs=p["qs"], ks=p["ks"], v8=p["v8"], vs=p["vs"], bm=p["bm"])
    d.update(over)
    return (d["q8"], d["k8"], d["qs"], d["ks"], d["v8"], d["vs"], d["bm"], scale)


U32 = 2.0 ** -24  # unit roundoff of f32


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_online_recurrence_without_p_rounding_equals_direct_softmax(reading):
    """Without the rounding of P both online recurrences give the direct softmax.  The plain
    reading works in fp64 throughout.  The kernel's reading forms c in f32 (at most 5 f32
    roundings: relative error 5u) and z - R with one f32 rounding (u |z - R|, |z - R| <=
    2 max|z| + 1), so each weight moves by a relative ln2 (7 max|z| + 1) u at most and a
    softmax average by 4 times that times max|v|."""
    p = _problem(3)
    out, _, _ = READINGS[reading](*_args(p, 0.25), round_p=False)
    if reading == "plain":
        assert np.allclose(out, _direct_softmax(p, 0.25), rtol=1e-11, atol=1e-12)
        return
    z = np.concatenate([(p["q8"][0, h].astype(np.int64) @ p["k8"][0, 0].astype(np.int64).T).ravel()
                        for h in range(p["q8"].shape[1])]).astype(np.float64)
    zmax = np.abs(z).max() * float(p["qs"].max()) * float(p["ks"].max()) * 0.25 / np.log(2.0)
    eps = np.log(2.0) * (7 * zmax + 1) * U32
    vmax = np.abs(formats.e4m3_decode(p["v8"]) * p["vs"][:, :, None, :]).max()
    assert np.all(np.abs(out - _direct_softmax(p, 0.25)) <= 4 * eps * vmax + 1e-12)


@pytest.mark.parametrize("seed,D,scale", [(10, 16, 0.5), (11, 64, 0.2), (12, 128, 128 ** -0.5)])
def test_power_of_two_reference_matches_final_max_up_to_subnormals(seed, D, scale):
    """The lazily moved power-of-two reference gives the codes of the order-free
    definition p8 = E4M3(2^(z - ceil(max z))) except where a weight falls in E4M3's
    subnormal range (below 2^-6) on one side: each such weight moves by at most the
    subnormal spacing 2^-9 (in units of the final reference), which bounds the output."""
    from oracle.formats import e4m3_decode, e4m3_encode
    p = _problem(seed, Nq=1, Nkv=1, Sq=128, Skv=1024, D=D, keep=1.0)
    got, _, _ = quant.qbsa_forward_pow2ref(*_args(p, scale))
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


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_loops_equal_vectorised_tiny(reading):
    p = _problem(4, Nq=2, Nkv=1, Sq=140, Skv=200, D=4, keep=1.0)
    # K grows block to block so that the running max moves at every block (the plain reading
    # rescales at each step; the power-of-two reference moves once the max passes R + 8)
    k8 = p["k8"].copy()
    k8[:, :, 128:] = np.clip(k8[:, :, 128:].astype(np.int64) * 3, -127, 127).astype(np.int8)
    a = READINGS[reading](*_args(p, 0.5, k8=k8))
    b = LOOPS[reading](*_args(p, 0.5, k8=k8))
    for x, y in zip(a, b):
        assert np.allclose(x, y, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_zero_query_gives_exact_counts_and_mean(reading):
    p = _problem(5)
    q8 = np.zeros_like(p["q8"])
    out, mx, sm = READINGS[reading](*_args(p, 0.25, q8=q8))
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


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_constant_v_returns_v_exactly(reading):
    p = _problem(6)
    v8 = np.full_like(p["v8"], 0x3B)            # 1.375 in every entry
    out, _, _ = READINGS[reading](*_args(p, 0.25, v8=v8))
    want = 1.375 * p["vs"][0, 0].astype(np.float64)
    assert np.allclose(out[0], np.broadcast_to(want, out[0].shape), rtol=1e-14, atol=0)


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_unkept_blocks_have_no_influence(reading):
    p = _problem(7, keep=0.5)
    a = READINGS[reading](*_args(p, 0.25))
    k8, v8 = p["k8"].copy(), p["v8"].copy()
    # blocks not kept by ANY query block of head 0 and 1 may be overwritten freely
    unused = np.nonzero(p["bm"][0].max(axis=(0, 1)) == 0)[0]
    assert len(unused) >= 0
    for kb in unused:
        k8[:, :, kb * 128:(kb + 1) * 128] = 99
        v8[:, :, kb * 128:(kb + 1) * 128] = 0x70
    b = READINGS[reading](*_args(p, 0.25, k8=k8, v8=v8))
    for x, y in zip(a, b):
        assert np.array_equal(x, y, equal_nan=True)


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_unkept_rows_are_zero(reading):
    p = _problem(8)
    bm = p["bm"].copy()
    bm[0, 1, 1, :] = 0
    out, mx, sm = READINGS[reading](*_args(p, 0.25, bm=bm))
    assert np.all(out[0, 1, 128:256] == 0) and np.all(mx[0, 1, 128:256] == -np.inf) and np.all(sm[0, 1, 128:256] == 0)


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_all_blocks_kept_tracks_unquantised_attention(reading):
    # quantisation error is small on N(0,1) data: loose sanity pin (the article gives no figure)
    p = _problem(9, Sq=256, Skv=256, D=64, keep=1.0)
    out, _, _ = READINGS[reading](*_args(p, 64 ** -0.5))
    ref, _, _ = dense.attention_forward(p["q"], p["k"], p["v"][:, [0, 0]], layout="BNSD", scale=64 ** -0.5)
    err = np.abs(out - ref)
    assert err.max() < 0.05 and err.mean() < 0.01


@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_block_mask_generator_counts_and_diagonal(keep):
    bm = block_keep_mask(3, 1, 4, 16, 16, keep)
    n = max(1, int(round(keep * 16)))
    assert np.all(bm.sum(axis=3) == n)
    assert np.all(bm[0, :, np.arange(16), np.arange(16)] == 1)


def test_fp16_then_e4m3_matches_torch_casts():
    """The weight's double rounding (FP16, then E4M3) against torch's float16 and
    float8_e4m3fn casts, on a dense grid of fp32 values in [2^-26, 448] (both signs) that
    includes the FP16 and E4M3 rounding midpoints and their neighbours."""
    import torch
    mant = np.arange(4096, dtype=np.float64) / 4096.0
    grid = [(1.0 + mant) * 2.0 ** e for e in range(-26, 9)]
    x = np.concatenate(grid + [np.random.default_rng(0).uniform(0, 448, 200000)])
    # E4M3 midpoints in every binade and FP16 midpoints around them, one fp32 ulp either side
    mids = []
    for e in range(-9, 9):
        for m in range(16):
            mids.append((1.0 + (m + 0.5) / 8.0) * 2.0 ** e)
            mids.append((1.0 + (m + 0.5) / 1024.0) * 2.0 ** e)
    mids = np.asarray(mids, dtype=np.float32)
    x = np.concatenate([x.astype(np.float32), mids, np.nextafter(mids, np.float32(0)),
                        np.nextafter(mids, np.float32(np.inf))])
    x = x[(x <= 448.0) & (x > 0)]
    x = np.concatenate([x, -x]).astype(np.float32)
    ours = formats.e4m3_encode(x.astype(np.float16).astype(np.float32))
    theirs = torch.from_numpy(x).to(torch.float16).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)
    # the grid tells the double rounding apart from a single rounding of the fp32 value
    assert np.sum(formats.e4m3_encode(x) != ours) > 0


def _fp8w(w):
    return formats.e4m3_decode(formats.e4m3_encode(w.astype(np.float16).astype(np.float32)))


def test_plain_reading_single_block_closed_form():
    """With one kept block per row the running max is the row max, so the plain reading is
    the closed form: p8 = E4M3(FP16(e^(s - max s))), O = Σ p8 v / Σ p8, sum = Σ p8."""
    p = _problem(13, Nq=2, Nkv=1, Sq=300, Skv=333, D=32, keep=1.0)
    rng = np.random.default_rng(13)
    bm = np.zeros_like(p["bm"])
    for h in range(2):
        for qb in range(3):
            bm[0, h, qb, rng.integers(0, 3)] = 1       # block 2 is the 77-key tail
    scale = 0.3
    out, mx, sm = quant.qbsa_forward(*_args(p, scale, bm=bm))
    vdq = formats.e4m3_decode(p["v8"][0, 0]) * p["vs"][0, 0][None, :]
    for h in range(2):
        for qb in range(3):
            kb = int(np.nonzero(bm[0, h, qb])[0][0])
            r0, r1, c0, c1 = qb * 128, min(300, qb * 128 + 128), kb * 128, min(333, kb * 128 + 128)
            t = p["q8"][0, h, r0:r1].astype(np.int64) @ p["k8"][0, 0, c0:c1].astype(np.int64).T
            s = t * (float(p["qs"][0, h, qb]) * float(p["ks"][0, 0, kb]) * scale)
            w8 = _fp8w(np.exp(s - s.max(axis=1, keepdims=True)))
            assert np.allclose(out[0, h, r0:r1], (w8 @ vdq[c0:c1]) / w8.sum(axis=1)[:, None], rtol=1e-12, atol=1e-13)
            assert np.allclose(sm[0, h, r0:r1], w8.sum(axis=1), rtol=1e-13)
            assert np.array_equal(mx[0, h, r0:r1], s.max(axis=1))


def test_plain_reading_max_in_first_block_closed_form():
    """When every row's maximum score lies in its first kept block the running max never
    moves afterwards, so over all kept blocks the plain reading equals the closed form with
    the row max: q = 1 everywhere and key 0 = 127 everywhere give key 0 the largest dot
    product for every query."""
    p = _problem(14, Nq=1, Nkv=1, Sq=200, Skv=600, D=16, keep=0.6)
    q8 = np.ones_like(p["q8"])
    k8 = p["k8"].copy()
    k8[0, 0, 0, :] = 127
    bm = p["bm"].copy()
    bm[0, 0, :, 0] = 1
    scale = 0.02
    out, mx, sm = quant.qbsa_forward(*_args(p, scale, q8=q8, k8=k8, bm=bm))
    vdq = formats.e4m3_decode(p["v8"][0, 0]) * p["vs"][0, 0][None, :]
    for qb in range(2):
        kept = np.nonzero(bm[0, 0, qb])[0]
        cols = np.concatenate([np.arange(kb * 128, min(600, kb * 128 + 128)) for kb in kept])
        ks_col = np.concatenate([np.full(min(600, kb * 128 + 128) - kb * 128, float(p["ks"][0, 0, kb]))
                                 for kb in kept])
        t = k8[0, 0, cols].astype(np.int64).sum(axis=1)                 # q = 1: t_j = Σ_c k8[j, c]
        s = t * float(p["qs"][0, 0, qb]) * ks_col * scale
        assert s.argmax() == 0
        w8 = _fp8w(np.exp(s - s.max()))
        r0, r1 = qb * 128, min(200, qb * 128 + 128)
        assert np.allclose(out[0, 0, r0:r1], ((w8 @ vdq[cols]) / w8.sum())[None, :], rtol=1e-12, atol=1e-13)
        assert np.allclose(sm[0, 0, r0:r1], w8.sum(), rtol=1e-13)


def _bound_problems():
    """Problems for the rounding-bound pins: a ragged GQA case, rows with a single 9-key
    tail block, and K growing block to block (the max moves many times per row)."""
    yield _problem(15, Nq=2, Nkv=1, Sq=300, Skv=400, D=64, keep=0.5), 64 ** -0.5
    p = _problem(16, Nq=2, Nkv=2, Sq=256, Skv=265, D=32, keep=0.5)
    bm = p["bm"].copy()
    bm[0, 0, 0] = 0
    bm[0, 0, 0, 2] = 1                               # only the 9-key tail block
    p["bm"] = bm
    yield p, -0.2
    p = _problem(17, Nq=1, Nkv=1, Sq=128, Skv=768, D=32, keep=1.0)
    k8 = p["k8"].astype(np.float64)
    for kb in range(6):
        k8[:, :, kb * 128:(kb + 1) * 128] *= (1 + kb) / 6.0
    p["k8"] = np.rint(k8).astype(np.int8)
    yield p, 0.4


@pytest.mark.parametrize("reading", sorted(READINGS))
def test_readings_within_rounding_bound_of_unrounded(reading):
    """Each reading's output lies within the per-weight E4M3 bound of the unrounded softmax:
    |O_r - O_w| <= G(center O_w) / A_r and |A_r - W| <= E (oracle.quant.qbsa_reading_gap_terms)."""
    for p, scale in _bound_problems():
        args = _args(p, scale)
        o_w, _, W = quant.qbsa_forward(*args, round_p=False)
        o_r, _, A = READINGS[reading](*args)
        G, E = quant.qbsa_reading_gap_terms(*args, center=o_w)
        live = A > 0
        assert np.all(np.abs(o_r - o_w)[live] <= (G / np.where(live, A, 1.0)[..., None])[live] + 1e-12)
        assert np.all(np.abs(A - W)[live] <= E[live] + 1e-12)


def test_pow2_reading_within_gap_bound_of_plain():
    """The power-of-two reading lies within the derived gap bound of the plain reading:
    |O_a - O_p| <= [G + W |O_w - O_p|] / A and |A - l_p| <= E + |W - l_p|."""
    for p, scale in _bound_problems():
        args = _args(p, scale)
        o_w, _, W = quant.qbsa_forward(*args, round_p=False)
        o_p, m_p, l_p = quant.qbsa_forward(*args)
        o_a, m_a, A = quant.qbsa_forward_pow2ref(*args)
        G, E = quant.qbsa_reading_gap_terms(*args, center=o_p)
        live = A > 0
        bound = (G + W[..., None] * np.abs(o_w - o_p)) / np.where(live, A, 1.0)[..., None]
        assert np.all(np.abs(o_a - o_p)[live] <= bound[live] + 1e-12)
        assert np.all(np.abs(A - l_p)[live] <= (E + np.abs(W - l_p))[live] + 1e-12)
        # the kernel's reading takes the block maximum as f32(t_max c) with c formed in f32:
        # at most 6 f32 roundings (relative 6u) from the exact maximum
        assert np.allclose(m_a[live], m_p[live], rtol=6 * U32 * 1.01, atol=1e-13)
