"""Ulysses sequence parallelism (heads <-> sequence all-to-all, head-chunked and block modes)
on two gloo ranks on CPU, against the oracle applied to the unsharded tensors.

The data movement is exact and the per-head attention is the fp64 oracle on both sides, so
every rank's output slice must equal the corresponding slice of the unsharded result bit for
bit, whatever the chunking."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, S, N, Nkv, D):
    from workloads import bf16_bits_to_f32, iid_normal_bf16
    f = lambda t, n: bf16_bits_to_f32(iid_normal_bf16(51, t, B, n, S, D)).astype(np.float64).transpose(0, 2, 1, 3)
    return f(0, N), f(1, Nkv), f(2, Nkv)  # BSND


def _oracle_bsnd(q, k, v, scale):
    """Unmasked attention of BSND float64 arrays, head h reading kv head h // (N / N_kv)."""
    from oracle import dense
    B, S, N, D = q.shape
    Skv, Nkv = k.shape[1], k.shape[2]
    out = np.zeros((B, S, N, v.shape[3]))
    ok = np.ones((S, Skv), dtype=bool)
    for b in range(B):
        for h in range(N):
            g = h // (N // Nkv)
            out[b, :, h] = dense.attend(q[b, :, h], k[b, :, g], v[b, :, g], scale, ok)[0]
    return out


def _rank_main(rank, world, port, case, out_q):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from quantized_block_sparse_attn_b200 import ulysses

    B, S, N, Nkv, D, comm_type, hpc, scale = case
    q, k, v = _inputs(B, S, N, Nkv, D)
    sl = slice(rank * S // world, (rank + 1) * S // world)

    def attn(qt, kt, vt):
        return torch.from_numpy(_oracle_bsnd(qt.numpy(), kt.numpy(), vt.numpy(), scale))

    got = ulysses.ulysses_attention(torch.from_numpy(q[:, sl].copy()), torch.from_numpy(k[:, sl].copy()),
                                    torch.from_numpy(v[:, sl].copy()), attn, comm_type=comm_type,
                                    heads_per_chunk=hpc)
    want = _oracle_bsnd(q, k, v, scale)[:, sl]
    out_q.put((rank, bool(np.array_equal(got.numpy(), want)), float(np.abs(got.numpy() - want).max())))
    dist.barrier()
    dist.destroy_process_group()


CASES = [
    # B, S, N, Nkv, D, comm_type, heads_per_chunk, scale
    (1, 64, 4, 4, 16, 0, None, 0.25),
    (2, 48, 8, 8, 8, 1, 2, 0.3),     # 2 chunks of 2 local heads
    (1, 64, 8, 4, 16, 1, 2, 0.25),   # GQA: 2 query heads per kv head
    (1, 40, 8, 8, 8, 2, 1, 0.3),     # 4 chunks, the local query split in 2 blocks
    (1, 64, 8, 2, 8, 2, 4, 0.2),     # GQA ratio 4, one chunk
]


@pytest.mark.parametrize("case", CASES)
def test_ulysses_matches_unsharded_attention(case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, equal, err in res:
        assert equal, f"rank {rank}: max error {err}"


def test_single_rank_is_the_plain_call():
    import datetime

    import torch
    import torch.distributed as dist
    from quantized_block_sparse_attn_b200 import ulysses

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=30))
    try:
        q, k, v = _inputs(1, 32, 4, 2, 8)
        attn = lambda a, b, c: torch.from_numpy(_oracle_bsnd(a.numpy(), b.numpy(), c.numpy(), 0.3))
        for ct, hpc in ((0, None), (1, 2), (2, 2)):
            got = ulysses.ulysses_attention(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn,
                                            comm_type=ct, heads_per_chunk=hpc)
            assert np.array_equal(got.numpy(), _oracle_bsnd(q, k, v, 0.3))
        with pytest.raises(ValueError):
            ulysses.ulysses_attention(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn,
                                      comm_type=1, heads_per_chunk=3)
    finally:
        dist.destroy_process_group()
