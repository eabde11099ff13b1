"""GPU parity of qbsa_fwd and the on-GPU quantisers against the oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import quantized_block_sparse_attn_b200 as qb
from oracle import dense, quant
from workloads import CONFIGS, block_keep_mask, blocky_qk_bf16, iid_normal_bf16, random_atten_mask, sample_rows
from oracle.formats import bf16_to_f64
from tests.gpu_util import QUANT_MAX_ABS, check_qbsa, compare_out, dev, dev_bf16, host_f64

pytestmark = pytest.mark.gpu


def _quantized(q, k, v):
    q8, qs = quant.quantize_qk_per_block(q)
    k8, ks = quant.quantize_qk_per_block(k)
    v8, vs = quant.quantize_v_per_channel(v)
    return q8, qs, k8, ks, v8, vs


def _run(q8, qs, k8, ks, v8, vs, bm, scale):
    out, smax, ssum = qb.qbsa_fwd(dev(q8), dev(k8), dev(qs), dev(ks), dev(v8), dev(vs), dev(bm), scale)
    qb.check()
    return host_f64(out), smax.cpu().numpy(), ssum.cpu().numpy()


@pytest.mark.parametrize("B,Nq,Nkv,Sq,Skv,keep", [
    (1, 2, 1, 300, 400, 0.5),     # ragged tails on both axes, GQA
    (1, 2, 2, 1024, 1024, 0.25),
    (2, 2, 1, 128, 640, 1.0),
    (1, 1, 1, 1, 129, 1.0),
])
def test_qbsa_parity_small(B, Nq, Nkv, Sq, Skv, keep):
    D = 128
    q = iid_normal_bf16(20, 0, B, Nq, Sq, D)
    k = iid_normal_bf16(20, 1, B, Nkv, Skv, D)
    v = iid_normal_bf16(20, 2, B, Nkv, Skv, D)
    q8, qs, k8, ks, v8, vs = _quantized(q, k, v)
    bm = block_keep_mask(20, B, Nq, -(-Sq // 128), -(-Skv // 128), keep)
    scale = D ** -0.5
    got, gmax, gsum = _run(q8, qs, k8, ks, v8, vs, bm, scale)
    check_qbsa(got, gmax, gsum, q8, k8, qs, ks, v8, vs, bm, scale, tag=f"{Sq}x{Skv} keep {keep}:")


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_qbsa_unequal_tile_pairs(sign):
    """Query blocks are processed in pairs: unequal kept counts, one side empty, an odd
    last pair, a ragged key tail; a negative scale exercises the row-minimum path."""
    B, Nq, Nkv, Sq, Skv, D = 1, 2, 1, 640, 700, 128
    nqb, nkb = 5, 6
    q = iid_normal_bf16(23, 0, B, Nq, Sq, D)
    k = iid_normal_bf16(23, 1, B, Nkv, Skv, D)
    v = iid_normal_bf16(23, 2, B, Nkv, Skv, D)
    q8, qs, k8, ks, v8, vs = _quantized(q, k, v)
    bm = (random_atten_mask(23, (B, Nq, nqb, nkb), 0.5) == 0).astype(np.uint8)
    bm[0, 0, 0, :] = 0          # pair 0 of head 0: first tile empty, second not
    bm[0, 0, 1, :] = 1
    bm[0, 0, 3, :] = 0          # pair 1 of head 0: second tile empty
    bm[0, 0, 2, :] = 0
    bm[0, 0, 2, 5] = 1          # ... first tile keeps only the ragged tail block
    bm[0, 1, 0, :] = 0
    bm[0, 1, 0, 2] = 1          # head 1, pair 0: 1 block against a full row
    bm[0, 1, 1, :] = 1
    scale = sign * D ** -0.5
    got, gmax, gsum = _run(q8, qs, k8, ks, v8, vs, bm, scale)
    check_qbsa(got, gmax, gsum, q8, k8, qs, ks, v8, vs, bm, scale, tag=f"unequal pairs sign {sign}:")


def _reference_moves(q8, qs, k8, ks, bm, scale, group):
    """Per (b, h, query row), the kept blocks at which the running max of z = t·c (log2 units)
    passes the power-of-two reference by more than 8 after the row's first block, i.e. where
    the kernel rescales O and L.  Returns (count of such events, events at a ragged last block)."""
    B, Nq, Sq, _ = q8.shape
    Skv = k8.shape[2]
    nkb = -(-Skv // 128)
    ragged = Skv % 128 != 0
    events = tail_events = 0
    for b in range(B):
        for h in range(Nq):
            g = h // group
            t_all = q8[b, h].astype(np.int64) @ k8[b, g].astype(np.int64).T  # [Sq, Skv]
            for qb_ in range(-(-Sq // 128)):
                rows = slice(qb_ * 128, min(Sq, (qb_ + 1) * 128))
                m = np.full(rows.stop - rows.start, -np.inf)
                ref = np.full_like(m, -np.inf)
                for kb in np.nonzero(bm[b, h, qb_])[0]:
                    cols = slice(kb * 128, min(Skv, (kb + 1) * 128))
                    c = qs[b, h, qb_] * ks[b, g, kb] * scale * np.log2(np.e)
                    z = t_all[rows, cols] * c
                    m = np.maximum(m, z.max(axis=1))
                    move = np.isfinite(ref) & (m > ref + 8)
                    events += int(move.sum())
                    if ragged and kb == nkb - 1:
                        tail_events += int(move.sum())
                    ref = np.where(~np.isfinite(ref) | (m > ref + 8), np.ceil(m), ref)
    return events, tail_events


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_qbsa_growing_keys_rescale_and_ragged_tail(sign):
    """Key blocks grow in magnitude (block j of K times 1 + 2 j before quantisation), so the
    running max of every row passes the power-of-two reference by more than 8 several times
    and O and L are rescaled in TMEM, also inside the out-of-line step of the ragged last key
    block; B = 2, GQA 4:2, ragged on both axes, some blocks dropped.  A negative scale runs
    the same through the row-minimum path."""
    from workloads import bf16_bits_from_f32, bf16_bits_to_f32
    B, Nq, Nkv, Sq, Skv, D = 2, 4, 2, 300, 1000, 128
    q = iid_normal_bf16(31, 0, B, Nq, Sq, D)
    kf = bf16_bits_to_f32(iid_normal_bf16(31, 1, B, Nkv, Skv, D)).copy()
    for j in range(-(-Skv // 128)):
        kf[:, :, j * 128:(j + 1) * 128] *= 1.0 + 2.0 * j
    k = bf16_bits_from_f32(kf)
    v = iid_normal_bf16(31, 2, B, Nkv, Skv, D)
    q8, qs, k8, ks, v8, vs = _quantized(q, k, v)
    nqb, nkb = -(-Sq // 128), -(-Skv // 128)
    bm = np.ones((B, Nq, nqb, nkb), dtype=np.uint8)
    bm[0, 1, :, 3] = 0
    bm[1, 2, 0, 1:5] = 0
    bm[1, 3, 2, :nkb - 1] = 0   # a row whose only block is the ragged one
    scale = sign * D ** -0.5
    events, tail_events = _reference_moves(q8, qs, k8, ks, bm, scale, Nq // Nkv)
    assert events > 1000 and tail_events > 100, (events, tail_events)
    got, gmax, gsum = _run(q8, qs, k8, ks, v8, vs, bm, scale)
    check_qbsa(got, gmax, gsum, q8, k8, qs, ks, v8, vs, bm, scale,
               tag=f"growing keys sign {sign} ({events} reference moves, {tail_events} in the ragged block):")


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_qbsa_more_units_than_sms(sign):
    """More (head, query-block pair) units than SMs, so the grid runs in several waves and
    CTAs start while others finish: ragged lengths, GQA, empty and unequal mask rows."""
    B, Nq, Nkv, Sq, Skv, D = 2, 40, 8, 1000, 777, 128
    nqb, nkb = 8, 7
    q = iid_normal_bf16(24, 0, B, Nq, Sq, D)
    k = iid_normal_bf16(24, 1, B, Nkv, Skv, D)
    v = iid_normal_bf16(24, 2, B, Nkv, Skv, D)
    q8, qs, k8, ks, v8, vs = _quantized(q, k, v)
    bm = (random_atten_mask(24, (B, Nq, nqb, nkb), 0.6) == 0).astype(np.uint8)
    bm[0, 3, :, :] = 0          # a head with no kept block at all
    bm[1, 7, 2, :] = 0
    scale = sign * D ** -0.5
    got, gmax, gsum = _run(q8, qs, k8, ks, v8, vs, bm, scale)
    check_qbsa(got, gmax, gsum, q8, k8, qs, ks, v8, vs, bm, scale, e4m3_flips=True, tag=f"waves sign {sign}:")


@pytest.mark.parametrize("chunks", [1, 3, 8])
def test_qbsa_host_buffers_pipelined(chunks):
    """Host tensors go through the chunked copy-in / compute / copy-out pipeline; each head's
    result must equal the single device launch bit for bit."""
    B, Nq, Nkv, Sq, Skv, D = 2, 8, 4, 512, 700, 128
    q = iid_normal_bf16(25, 0, B, Nq, Sq, D)
    k = iid_normal_bf16(25, 1, B, Nkv, Skv, D)
    v = iid_normal_bf16(25, 2, B, Nkv, Skv, D)
    q8, qs, k8, ks, v8, vs = _quantized(q, k, v)
    bm = block_keep_mask(25, B, Nq, 4, 6, 0.5)
    host = [torch.from_numpy(np.ascontiguousarray(x)) for x in (q8, k8, qs, ks, v8, vs, bm)]
    got = qb.qbsa_fwd(*host, 0.09, host_chunks=chunks)
    qb.check()
    want = qb.qbsa_fwd(*[h.cuda() for h in host], 0.09)
    qb.check()
    for g, w in zip(got, want):
        assert not g.is_cuda and g.is_pinned()
        assert torch.equal(g, w.cpu())


def test_qbsa_short_loops_repeated():
    """Two or three kept blocks per query block, repeated: the last-P·V wait must not pass early."""
    D = 128
    for rep in range(6):
        for S in (256, 384):
            q = iid_normal_bf16(40 + rep, 0, 1, 1, S, D)
            k = iid_normal_bf16(40 + rep, 1, 1, 1, S, D)
            v = iid_normal_bf16(40 + rep, 2, 1, 1, S, D)
            q8, qs, k8, ks, v8, vs = _quantized(q, k, v)
            bm = np.ones((1, 1, S // 128, S // 128), dtype=np.uint8)
            got, gmax, gsum = _run(q8, qs, k8, ks, v8, vs, bm, D ** -0.5)
            check_qbsa(got, gmax, gsum, q8, k8, qs, ks, v8, vs, bm, D ** -0.5, tag=f"S={S} rep {rep}:")


def test_qbsa_empty_rows_and_zero_query_counts():
    """q = 0 gives p8 = 1 for every kept key: softmax_sum must be the exact kept-column count."""
    B, Nq, Nkv, Sq, Skv, D = 1, 2, 1, 384, 333, 128
    k = iid_normal_bf16(21, 1, B, Nkv, Skv, D)
    v = iid_normal_bf16(21, 2, B, Nkv, Skv, D)
    k8, ks = quant.quantize_qk_per_block(k)
    v8, vs = quant.quantize_v_per_channel(v)
    q8 = np.zeros((B, Nq, Sq, D), dtype=np.int8)
    qs = np.ones((B, Nq, 3), dtype=np.float32)
    bm = block_keep_mask(21, B, Nq, 3, 3, 0.67)
    bm[0, 1, 2, :] = 0  # a query block with no kept key block
    got, gmax, gsum = _run(q8, qs, k8, ks, v8, vs, bm, 0.1)
    for h in range(Nq):
        for qb_ in range(3):
            cols = sum(min(Skv, kb * 128 + 128) - kb * 128 for kb in np.nonzero(bm[0, h, qb_])[0])
            assert np.all(gsum[0, h, qb_ * 128:(qb_ + 1) * 128] == np.float32(cols))
            if cols == 0:
                assert np.all(got[0, h, qb_ * 128:(qb_ + 1) * 128] == 0)
                assert np.all(np.isneginf(gmax[0, h, qb_ * 128:(qb_ + 1) * 128]))
            else:
                assert np.all(gmax[0, h, qb_ * 128:(qb_ + 1) * 128] == 0)


def test_block_lists_hook_bit_exact():
    rng = np.random.default_rng(22)
    for n_kb in (1, 31, 32, 33, 512, 2048):
        rows = (rng.random((9, n_kb)) < 0.3).astype(np.uint8)
        rows[0] = 0
        rows[1] = 1
        lists, counts = qb.block_lists(dev(rows))
        lists, counts = lists.cpu().numpy(), counts.cpu().numpy()
        for r in range(9):
            idx = np.nonzero(rows[r])[0]
            assert counts[r] == len(idx)
            assert np.array_equal(lists[r, :len(idx)], idx)
            assert np.all(lists[r, len(idx):] == -1)


@pytest.mark.parametrize("B,N,S,D", [
    (2, 3, 300, 128),       # ragged 128-row block; V: one chunk per head
    (2, 3, 4096, 128),      # V: 16 chunks per head, pass 2 of a head interleaved with pass 1 of the next
    (1, 1, 100, 128),       # a single head and a single short chunk
    (1, 5, 1000, 64),
    (3, 2, 777, 256),
    (1, 2, 40000, 128),     # 157 chunks per head, ragged last chunk
])
def test_quantisers_bit_exact(B, N, S, D):
    x = blocky_qk_bf16(23, "q", B, N, S, D)
    v = iid_normal_bf16(23, 2, B, N, S, D)
    v[0, N - 1, :, 5] = 0  # an all-zero channel takes scale 1
    c8, cs = qb.quantize_qk(dev_bf16(x))
    v8, vs = qb.quantize_v(dev_bf16(v))
    qb.check()
    r8, rs = quant.quantize_qk_per_block(x)
    rv8, rvs = quant.quantize_v_per_channel(v)
    assert np.array_equal(c8.cpu().numpy(), r8)
    assert np.array_equal(cs.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(vs.cpu().numpy().view(np.uint32), rvs.view(np.uint32))
    assert np.array_equal(v8.cpu().numpy(), rv8)


def test_quantise_v_repeated_calls():
    """The V quantiser's scratch (ticket, arrival counters, column maxima) starts from zero on
    every call: the same input twice, then a different one, give the oracle's bytes each time."""
    B, N, S, D = 1, 4, 3000, 128
    v1 = iid_normal_bf16(26, 2, B, N, S, D)
    v2 = iid_normal_bf16(27, 2, B, N, S, D)
    for v in (v1, v1, v2):
        v8, vs = qb.quantize_v(dev_bf16(v))
        qb.check()
        rv8, rvs = quant.quantize_v_per_channel(v)
        assert np.array_equal(v8.cpu().numpy(), rv8)
        assert np.array_equal(vs.cpu().numpy().view(np.uint32), rvs.view(np.uint32))


def _qbsa_workload(S, keep, heads_for_oracle, n_qblocks):
    """One point of the Fig 4.1 workload (B=1, N=40, D=128), quantised on the GPU; sampled
    heads and query blocks (first and last included) against both oracle readings."""
    c = CONFIGS["qbsa"]
    N, D, seed = c["Nq"], c["D"], c["seed"]
    q = blocky_qk_bf16(seed, "q", 1, N, S, D)
    k = blocky_qk_bf16(seed, "k", 1, N, S, D)
    v = iid_normal_bf16(seed, 2, 1, N, S, D)
    nb = S // 128
    bm = block_keep_mask(seed, 1, N, nb, nb, keep)
    # GPU path: quantise on the GPU (checked bit-exact against the oracle on the sampled heads)
    tq8, tqs = qb.quantize_qk(dev_bf16(q))
    tk8, tks = qb.quantize_qk(dev_bf16(k))
    tv8, tvs = qb.quantize_v(dev_bf16(v))
    out, smax, ssum = qb.qbsa_fwd(tq8, tk8, tqs, tks, tv8, tvs, dev(bm), c["scale"])
    qb.check()
    got, gmax, gsum = host_f64(out), smax.cpu().numpy(), ssum.cpu().numpy()
    qbs = sample_rows(seed, S, n_qblocks)
    assert 0 in qbs and nb - 1 in qbs
    for h in heads_for_oracle:
        sl = (slice(0, 1), slice(h, h + 1))
        q8, qs, k8, ks, v8, vs = _quantized(q[sl], k[sl], v[sl])
        assert np.array_equal(tq8[0, h].cpu().numpy(), q8[0, 0])
        assert np.array_equal(tk8[0, h].cpu().numpy(), k8[0, 0])
        assert np.array_equal(tv8[0, h].cpu().numpy(), v8[0, 0])
        assert np.array_equal(tqs[0, h].cpu().numpy().view(np.uint32), qs[0, 0].view(np.uint32))
        assert np.array_equal(tks[0, h].cpu().numpy().view(np.uint32), ks[0, 0].view(np.uint32))
        assert np.array_equal(tvs[0, h].cpu().numpy().view(np.uint32), vs[0, 0].view(np.uint32))
        check_qbsa(got[:, h:h + 1], gmax[:, h:h + 1], gsum[:, h:h + 1], q8, k8, qs, ks, v8, vs, bm[:, h:h + 1],
                   c["scale"], q_blocks=qbs, plain_max_abs=QUANT_MAX_ABS, tag=f"S={S} keep={keep} head {h}:")
        # reported, not gated: error against the unquantised bf16 attention over the same kept blocks
        rows = np.concatenate([np.arange(b_ * 128, b_ * 128 + 128) for b_ in qbs])
        ok = np.repeat(bm[0, h][qbs], 128, axis=0)
        ok = np.repeat(ok, 128, axis=1).astype(bool)
        dref, _, _ = dense.attend(bf16_to_f64(q[0, h, rows]), bf16_to_f64(k[0, h]), bf16_to_f64(v[0, h]),
                                  c["scale"], ok)
        e = np.abs(got[0, h, rows] - dref)
        print(f"S={S} keep={keep} head {h}: error vs unquantised attention max {e.max():.3e} mean {e.mean():.3e}")


# The ten points of the Fig 4.1 range (S from 8K to 128K, sparsity 0.9 and 0.5)
@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_qbsa_workload_8k_sampled(keep):
    _qbsa_workload(8192, keep, heads_for_oracle=[0, 39], n_qblocks=6)


@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_qbsa_workload_16k_sampled(keep):
    _qbsa_workload(16384, keep, heads_for_oracle=[0, 17], n_qblocks=4)


@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_qbsa_workload_32k_sampled(keep):
    _qbsa_workload(32768, keep, heads_for_oracle=[5, 39], n_qblocks=3)


@pytest.mark.slow
@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_qbsa_workload_64k_sampled(keep):
    _qbsa_workload(65536, keep, heads_for_oracle=[0, 21], n_qblocks=3)


@pytest.mark.slow
@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_qbsa_workload_128k_sampled(keep):
    """The largest configuration of the workload: S = 128K."""
    _qbsa_workload(131072, keep, heads_for_oracle=[7], n_qblocks=2)
