"""Ulysses attention on the GPU with this library's attn_fwd kernel on one NCCL rank: every
all_to_all_single of the heads <-> sequence exchange runs through NCCL (with one rank it moves
the data to itself), the head chunks, query blocks and side-stream exchange run as in a
multi-GPU job.  Every mode must reproduce one direct attn_fwd call bit for bit (the kernel
computes each (head, query row) independently of the others) and match the fp64 oracle on
sampled heads.  The exchange between two or more ranks is tested on gloo CPU ranks."""

import datetime
import os
import socket

import pytest
import torch

import quantized_block_sparse_attn_b200 as qb
from quantized_block_sparse_attn_b200 import ulysses
from oracle import dense
from oracle.formats import bf16_to_f64
from workloads import iid_normal_bf16
from tests.gpu_util import DENSE_MAX_ABS, DENSE_MEAN_ABS, compare_out, dev_bf16, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield dist
    dist.destroy_process_group()


@pytest.mark.parametrize("N,Nkv,comm_type,hpc", [(8, 8, 0, None), (8, 8, 1, 2), (8, 4, 1, 4), (8, 8, 2, 2), (8, 2, 2, 4)])
def test_ulysses_single_rank_matches_direct_call(nccl_group, N, Nkv, comm_type, hpc):
    B, S, D = 1, 512, 128
    scale = D ** -0.5
    hq, hk, hv = (iid_normal_bf16(52, 0, B, N, S, D), iid_normal_bf16(52, 1, B, Nkv, S, D),
                  iid_normal_bf16(52, 2, B, Nkv, S, D))
    q = dev_bf16(hq).transpose(1, 2).contiguous()   # BSND
    k = dev_bf16(hk).transpose(1, 2).contiguous()
    v = dev_bf16(hv).transpose(1, 2).contiguous()
    want, _, _ = qb.attn_fwd(q, k, v, N, "BSND", scale=scale, return_stats=False)
    got = ulysses.ulysses_attention(q, k, v, ulysses.bsnd_attention(scale), comm_type=comm_type,
                                    heads_per_chunk=hpc)
    torch.cuda.synchronize()
    qb.check()
    assert torch.equal(got, want)
    out = host_f64(got)                                               # BSND
    ok = torch.ones((S, S), dtype=torch.bool).numpy()
    for h in (0, N - 1):
        g = h // (N // Nkv)
        ref, _, _ = dense.attend(bf16_to_f64(hq[0, h]), bf16_to_f64(hk[0, g]), bf16_to_f64(hv[0, g]), scale, ok)
        compare_out(out[0, :, h], ref, DENSE_MAX_ABS, DENSE_MEAN_ABS)


def test_ulysses_exchange_round_trip_through_nccl(nccl_group):
    """heads_to_sequence then sequence_to_heads through NCCL returns the input bit for bit."""
    x = torch.randn(2, 64, 8, 128, device="cuda", dtype=torch.bfloat16)
    y = ulysses.heads_to_sequence(x)
    assert y.data_ptr() != x.data_ptr() and torch.equal(y, x)
    z = ulysses.sequence_to_heads(y)
    torch.cuda.synchronize()
    assert torch.equal(z, x)
