"""GPU parity of attn_fwd (dense bf16) against the fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import quantized_block_sparse_attn_b200 as qb
from oracle import dense
from workloads import (CONFIGS, bf16_bits_from_f32, blocky_qk_bf16, iid_normal_bf16, random_atten_mask,
                       random_pse_bf16, sample_rows)
from tests.gpu_util import (DENSE_MAX_ABS, DENSE_MEAN_ABS, compare_out, compare_stats, dev, dev_bf16, host_f64)

pytestmark = pytest.mark.gpu
INF = qb.INF_TOKENS


def _bnsd(seed, B, Nq, Nkv, Sq, Skv, D):
    q = iid_normal_bf16(seed, 0, B, Nq, Sq, D)
    k = iid_normal_bf16(seed, 1, B, Nkv, Skv, D)
    v = iid_normal_bf16(seed, 2, B, Nkv, Skv, D)
    return q, k, v


def _run_and_compare(q, k, v, layout, Nq, scale, mode=0, pre=INF, nxt=INF, mask=None, mask_shape=None, pse=None,
                     cq=None, ck=None, q_rows=None, heads=None):
    tq, tk, tv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    tm = None if mask is None else dev(mask)
    tp = None if pse is None else dev_bf16(pse)
    out, smax, ssum = qb.attn_fwd(tq, tk, tv, Nq, layout, atten_mask=tm, mask_shape=mask_shape, pse=tp, scale=scale,
                                  sparse_mode=mode, pre_tokens=pre, next_tokens=nxt, actual_seq_qlen=cq,
                                  actual_seq_kvlen=ck)
    qb.check()
    ref, rmax, rsum = dense.attention_forward(q, k, v, layout=layout, scale=scale, sparse_mode=mode, pre_tokens=pre,
                                              next_tokens=nxt, atten_mask=mask, pse=pse, actual_seq_qlen=cq,
                                              actual_seq_kvlen=ck, q_rows=q_rows, heads=heads)
    mx, mn = compare_out(host_f64(out), ref, DENSE_MAX_ABS, DENSE_MEAN_ABS)
    compare_stats(smax.cpu().numpy(), ssum.cpu().numpy(), rmax, rsum)
    print(f"{layout} Sq={q.shape[2] if layout == 'BNSD' else q.shape[1] if layout == 'BSND' else q.shape[0]} "
          f"mode {mode}: max abs err {mx:.3e}, mean abs err {mn:.3e}")
    return mx, mn


@pytest.mark.parametrize("B,Nq,Nkv,Sq,Skv,D,mode,pre,nxt,layout", [
    (1, 2, 2, 256, 256, 64, 0, INF, INF, "BNSD"),      # the tiny workload
    (2, 4, 2, 300, 333, 128, 0, INF, INF, "BNSD"),     # ragged tails, GQA
    (1, 2, 1, 300, 333, 128, 2, INF, INF, "BNSD"),
    (1, 2, 1, 333, 300, 128, 3, INF, INF, "BNSD"),     # rows with no key (Skv < Sq)
    (1, 2, 2, 300, 333, 128, 3, INF, INF, "BSND"),
    (2, 2, 1, 520, 520, 64, 0, 100, 20, "BSND"),       # band
    (1, 1, 1, 640, 640, 128, 0, -50, 200, "BNSD"),     # band excluding the diagonal
    (1, 1, 1, 1, 1, 128, 0, INF, INF, "BNSD"),
    # unmasked D = 128 (two query tiles per CTA): BSND, an odd tile count, one short K tile
    (1, 3, 1, 650, 333, 128, 0, INF, INF, "BSND"),
    (2, 2, 2, 129, 100, 128, 0, INF, INF, "BNSD"),
    (1, 1, 1, 1, 700, 64, 3, INF, INF, "BNSD"),
    (1, 3, 1, 1000, 1000, 128, 2, INF, INF, "BNSD"),
    # masked two-tile kernel (per-tile K ranges)
    (1, 2, 1, 600, 600, 128, 0, 0, 0, "BNSD"),         # diagonal-only band: one K tile per query tile
    (1, 2, 2, 1000, 300, 128, 3, INF, INF, "BSND"),    # most rows have no key
    (2, 3, 1, 257, 1029, 128, 2, INF, INF, "BNSD"),    # top-left causal with S_kv > S_q
])
def test_dense_parity(B, Nq, Nkv, Sq, Skv, D, mode, pre, nxt, layout):
    q, k, v = _bnsd(7, B, Nq, Nkv, Sq, Skv, D)
    if layout == "BSND":
        q, k, v = (np.ascontiguousarray(np.swapaxes(t, 1, 2)) for t in (q, k, v))
    _run_and_compare(q, k, v, layout, Nq, D ** -0.5, mode, pre, nxt)


def test_dense_short_k_loops_repeated():
    """Two to three K tiles per CTA, repeated: the last-P·V wait must not pass early."""
    for rep in range(8):
        for S, D in ((256, 64), (256, 128), (384, 64), (384, 128)):
            q, k, v = _bnsd(30 + rep, 1, 1, 1, S, S, D)
            _run_and_compare(q, k, v, "BNSD", 1, D ** -0.5)


@pytest.mark.parametrize("shape", ["SS", "B1SS", "BNSS"])
def test_dense_atten_mask(shape):
    B, Nq, S, D = 2, 2, 200, 64
    q, k, v = _bnsd(8, B, Nq, Nq, S, S, D)
    mshape = {"SS": (S, S), "B1SS": (B, 1, S, S), "BNSS": (B, Nq, S, S)}[shape]
    mask = random_atten_mask(8, mshape, 0.3)
    _run_and_compare(q, k, v, "BNSD", Nq, 0.125, 0, 150, 150, mask=mask, mask_shape=shape)


@pytest.mark.parametrize("bcast", [False, True])
def test_dense_pse(bcast):
    B, Nq, S, D = 2, 2, 200, 128
    q, k, v = _bnsd(9, B, Nq, Nq, S, S, D)
    pse = random_pse_bf16(9, (1 if bcast else B, Nq, S, S), 2.0)
    _run_and_compare(q, k, v, "BNSD", Nq, D ** -0.5, 3, pse=pse)


@pytest.mark.parametrize("shape", ["SS", "B1SS", "BNSS"])
@pytest.mark.parametrize("D", [64, 128])
def test_dense_atten_mask_aligned_rows(shape, D):
    """S_kv % 16 == 0: the mask rows are read as 16-byte vectors a key tile ahead, except the
    half-tiles that run past S_kv (384..399 here), which are read byte by byte."""
    B, Nq, Sq, Skv = 2, 2, 300, 400
    q, k, v = _bnsd(18, B, Nq, Nq, Sq, Skv, D)
    mshape = {"SS": (Sq, Skv), "B1SS": (B, 1, Sq, Skv), "BNSS": (B, Nq, Sq, Skv)}[shape]
    mask = random_atten_mask(18, mshape, 0.4)
    _run_and_compare(q, k, v, "BNSD", Nq, D ** -0.5, 0, 200, 150, mask=mask, mask_shape=shape)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Skv", [16, 96])
def test_dense_mask_and_pse_short_keys(Skv, D):
    """S_kv below one key tile but 16-byte aligned: the staged mask / pse boxes extend past the
    rows (the copy fills the rest, which the S_kv bound masks)."""
    B, Nq, Sq = 2, 2, 130
    q, k, v = _bnsd(20, B, Nq, Nq, Sq, Skv, D)
    pse = random_pse_bf16(20, (1, Nq, Sq, Skv), 1.0)
    mask = random_atten_mask(20, (B, Nq, Sq, Skv), 0.3)
    _run_and_compare(q, k, v, "BNSD", Nq, D ** -0.5, 0, mask=mask, mask_shape="BNSS", pse=pse)


@pytest.mark.parametrize("Skv", [400, 403, 408])
def test_dense_pse_and_mask_together(Skv):
    """pse and atten_mask in one call: both staged by TMA (S_kv = 400), neither (S_kv = 403:
    rows not 16-byte aligned, read element by element), or only pse (S_kv = 408: pse rows
    16-byte aligned, mask rows not)."""
    B, Nq, Sq, D = 1, 2, 260, 128
    q, k, v = _bnsd(19, B, Nq, Nq, Sq, Skv, D)
    pse = random_pse_bf16(19, (B, Nq, Sq, Skv), 2.0)
    mask = random_atten_mask(19, (Sq, Skv), 0.3)
    _run_and_compare(q, k, v, "BNSD", Nq, D ** -0.5, 0, mask=mask, mask_shape="SS", pse=pse)


@pytest.mark.parametrize("D", [64, 128])
def test_dense_tnd_gqa_causal(D):
    lens_q, lens_k = [100, 300, 77, 256], [130, 300, 50, 256]
    cq, ck = np.cumsum(lens_q), np.cumsum(lens_k)
    Nq, Nkv = 4, 2
    q = iid_normal_bf16(10, 0, 1, 1, cq[-1], Nq * D).reshape(cq[-1], Nq, D)
    k = iid_normal_bf16(10, 1, 1, 1, ck[-1], Nkv * D).reshape(ck[-1], Nkv, D)
    v = iid_normal_bf16(10, 2, 1, 1, ck[-1], Nkv * D).reshape(ck[-1], Nkv, D)
    _run_and_compare(q, k, v, "TND", Nq, D ** -0.5, 3, cq=cq, ck=ck)


@pytest.mark.parametrize("mode,pre,nxt,layout", [(0, 300, 40, "BNSD"), (2, INF, INF, "BNSD"), (3, INF, INF, "BSND"),
                                                 (3, INF, INF, "TND"), (0, INF, INF, "BNSD"), (0, INF, INF, "BSND")])
def test_mask_logic_bit_exact_via_zero_query(mode, pre, nxt, layout):
    """Q = 0 makes every kept weight exactly 1: softmax_sum must equal the kept-key count."""
    D, Nq, Nkv = 128, 2, 1
    if layout == "TND":
        lens_q, lens_k = [333, 129, 500], [400, 129, 257]
        cq, ck = np.cumsum(lens_q), np.cumsum(lens_k)
        q = np.zeros((cq[-1], Nq, D), dtype=np.uint16)
        k = iid_normal_bf16(11, 1, 1, 1, ck[-1], Nkv * D).reshape(ck[-1], Nkv, D)
        v = iid_normal_bf16(11, 2, 1, 1, ck[-1], Nkv * D).reshape(ck[-1], Nkv, D)
    else:
        cq = ck = None
        Sq, Skv = 700, 531
        q = np.zeros((1, Nq, Sq, D), dtype=np.uint16)
        _, k, v = _bnsd(11, 1, Nq, Nkv, Sq, Skv, D)
        if layout == "BSND":
            q, k, v = (np.ascontiguousarray(np.swapaxes(t, 1, 2)) for t in (q, k, v))
    out, smax, ssum = qb.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), Nq, layout, scale=0.3, sparse_mode=mode,
                                  pre_tokens=pre, next_tokens=nxt, actual_seq_qlen=cq, actual_seq_kvlen=ck)
    qb.check()
    ssum = ssum.cpu().numpy()
    if layout == "TND":
        for b in range(len(cq)):
            q0, q1 = (cq[b - 1] if b else 0), cq[b]
            cnt = dense.allowed(q1 - q0, lens_k[b], mode, pre, nxt).sum(axis=1)
            for h in range(Nq):
                assert np.array_equal(ssum[h, q0:q1], cnt.astype(np.float32))
    else:
        cnt = dense.allowed(700, 531, mode, pre, nxt).sum(axis=1)
        for h in range(Nq):
            assert np.array_equal(ssum[0, h], cnt.astype(np.float32))


def test_causal_workload_sampled():
    c = CONFIGS["causal"]
    B, N, S, D = c["B"], c["Nq"], c["S"], c["D"]
    q, k, v = _bnsd(c["seed"], B, N, N, S, S, D)
    rows = np.concatenate([np.arange(qb_ * 128, qb_ * 128 + 128) for qb_ in sample_rows(c["seed"], S, 4)])
    _run_and_compare(q, k, v, "BNSD", N, c["scale"], 3, q_rows=rows)


def test_gqa_varlen_workload_sampled():
    c = CONFIGS["gqa_varlen"]
    lens = list(c["seqlens"])
    cq = np.cumsum(lens)
    T, Nq, Nkv, D = cq[-1], c["Nq"], c["Nkv"], c["D"]
    q = iid_normal_bf16(c["seed"], 0, 1, 1, T, Nq * D).reshape(T, Nq, D)
    k = iid_normal_bf16(c["seed"], 1, 1, 1, T, Nkv * D).reshape(T, Nkv, D)
    v = iid_normal_bf16(c["seed"], 2, 1, 1, T, Nkv * D).reshape(T, Nkv, D)
    rows = np.array(sorted(set(range(0, 128)) | set(range(1000, 1024)) | set(range(4000, 4100)) |
                           set(range(10232, 10360))))
    _run_and_compare(q, k, v, "TND", Nq, c["scale"], 3, cq=cq, ck=cq, q_rows=rows, heads=None)


@pytest.mark.slow
def test_video_workload_sampled():
    c = CONFIGS["video"]
    N, S, D = c["Nq"], c["S"], c["D"]
    heads = [0, 17, 39]
    q = blocky_qk_bf16(c["seed"], "q", 1, N, S, D)
    k = blocky_qk_bf16(c["seed"], "k", 1, N, S, D)
    v = iid_normal_bf16(c["seed"], 2, 1, N, S, D)
    rows = np.concatenate([np.arange(b * 128, b * 128 + 128) for b in sample_rows(c["seed"], S, 4)])
    _run_and_compare(q, k, v, "BNSD", N, c["scale"], 0, q_rows=rows, heads=[(0, h) for h in heads])


@pytest.mark.parametrize("B,Nq,Nkv,S,D,keep", [(1, 2, 1, 300, 128, 0.5), (2, 2, 2, 1024, 64, 0.25),
                                               (1, 3, 1, 640, 128, 1.0), (2, 4, 2, 2048, 128, 0.3)])
def test_bsa_parity(B, Nq, Nkv, S, D, keep):
    """bf16 block-sparse attention = the dense oracle with the unkept blocks masked."""
    from workloads import block_keep_mask
    q, k, v = _bnsd(12, B, Nq, Nkv, S, S, D)
    nb = -(-S // 128)
    bm = block_keep_mask(12, B, Nq, nb, nb, keep)
    bm[0, 0, 1 % nb, :] = 0  # one query tile with no kept block
    out, smax, ssum = qb.bsa_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev(bm), D ** -0.5)
    qb.check()
    el = np.repeat(np.repeat(bm, 128, axis=2), 128, axis=3)[:, :, :S, :S]
    ref, rmax, rsum = dense.attention_forward(q, k, v, layout="BNSD", scale=D ** -0.5,
                                              atten_mask=(el == 0).astype(np.uint8))
    compare_out(host_f64(out), ref, DENSE_MAX_ABS, DENSE_MEAN_ABS)
    compare_stats(smax.cpu().numpy(), ssum.cpu().numpy(), rmax, rsum)


def _quarter(v):
    """V / 4 (exact in bf16).  With the sharp rows of a growing K an output is close to one
    key's value, so |O| reaches the largest |v|; bf16 rounding of P and of the output then
    costs up to 2^-8 |O| each, which exceeds 1e-2 at |O| ~ 4 even for exact arithmetic.  A
    quarter of V keeps |O| <= ~1 and the rescale path under the dense tolerance."""
    from workloads import bf16_bits_to_f32
    return bf16_bits_from_f32(bf16_bits_to_f32(v) * np.float32(0.25))


def _growing_k(k, Skv, factor=3.0):
    """K tile j (128 keys) multiplied by 1 + factor * j.  With iid N(0,1) data and scale
    D^-0.5 a row's max then grows by a median of about 11 log2 units per tile, past the
    kernels' lazy-rescale threshold of 8: on the first test case every row rescales O in
    TMEM at two to five of its tiles (3.3 on average)."""
    from workloads import bf16_bits_to_f32
    kf = bf16_bits_to_f32(k).copy()
    for j in range(-(-Skv // 128)):
        kf[:, :, j * 128:(j + 1) * 128] *= 1.0 + factor * j
    return bf16_bits_from_f32(kf)


@pytest.mark.parametrize("B,Nq,Nkv,Sq,Skv,D,mode,layout", [
    (1, 2, 2, 256, 680, 128, 0, "BNSD"),    # two-tile kernel, one pair per head, short last K tile
    (1, 3, 1, 650, 680, 128, 0, "BSND"),    # two-tile kernel, odd tile count
    (1, 2, 1, 300, 680, 64, 0, "BNSD"),     # one-tile kernel (D = 64)
    (1, 2, 1, 300, 680, 128, 3, "BNSD"),    # masked two-tile kernel, causal (bottom-right): unequal K ranges
])
def test_dense_lazy_rescale_growing_k(B, Nq, Nkv, Sq, Skv, D, mode, layout):
    """The rescale of O in TMEM (taken only when the running max grows by more than 2^8)
    against the oracle, with every row's max growing past that threshold several times."""
    q, k, v = _bnsd(13, B, Nq, Nkv, Sq, Skv, D)
    k, v = _growing_k(k, Skv), _quarter(v)
    if layout == "BSND":
        q, k, v = (np.ascontiguousarray(np.swapaxes(t, 1, 2)) for t in (q, k, v))
    _run_and_compare(q, k, v, layout, Nq, D ** -0.5, mode)


@pytest.mark.parametrize("D", [64, 128])
def test_dense_lazy_rescale_growing_k_mask_and_pse(D):
    """The one-tile kernel's atten_mask / pse instantiation through the same rescales: S_kv =
    688 (a multiple of 16, so all but the last half-tile are read as vectors)."""
    B, Nq, Nkv, Sq, Skv = 1, 2, 1, 300, 688
    q, k, v = _bnsd(15, B, Nq, Nkv, Sq, Skv, D)
    k, v = _growing_k(k, Skv), _quarter(v)
    mask = random_atten_mask(15, (B, 1, Sq, Skv), 0.2)
    pse = random_pse_bf16(15, (B, Nq, Sq, Skv), 0.5)
    _run_and_compare(q, k, v, "BNSD", Nq, D ** -0.5, 0, mask=mask, mask_shape="B1SS", pse=pse)


def test_bsa_lazy_rescale_growing_k():
    """bsa_fwd (one-tile kernel walking a kept-block list) with the row max growing past the
    rescale threshold at several kept K tiles."""
    from workloads import block_keep_mask
    B, Nq, Nkv, S, D = 1, 2, 1, 640, 128
    q, k, v = _bnsd(14, B, Nq, Nkv, S, S, D)
    k, v = _growing_k(k, S), _quarter(v)
    bm = block_keep_mask(14, B, Nq, 5, 5, 0.6)
    out, smax, ssum = qb.bsa_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev(bm), D ** -0.5)
    qb.check()
    el = np.repeat(np.repeat(bm, 128, axis=2), 128, axis=3)
    ref, rmax, rsum = dense.attention_forward(q, k, v, layout="BNSD", scale=D ** -0.5,
                                              atten_mask=(el == 0).astype(np.uint8))
    compare_out(host_f64(out), ref, DENSE_MAX_ABS, DENSE_MEAN_ABS)
    compare_stats(smax.cpu().numpy(), ssum.cpu().numpy(), rmax, rsum)
