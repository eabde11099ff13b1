"""Ulysses attention on the GPU with this library's attn_fwd kernel: one NCCL rank (the data
exchange is the identity, the head chunks, query blocks and side-stream exchange run as in
a multi-GPU job); every mode must reproduce one direct attn_fwd call bit for bit, since the
kernel computes each (head, query row) independently of the others."""

import datetime
import os
import socket

import pytest
import torch

import quantized_block_sparse_attn_b200 as qb
from quantized_block_sparse_attn_b200 import ulysses
from workloads import iid_normal_bf16
from tests.gpu_util import dev_bf16

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
    q = dev_bf16(iid_normal_bf16(52, 0, B, N, S, D)).transpose(1, 2).contiguous()   # BSND
    k = dev_bf16(iid_normal_bf16(52, 1, B, Nkv, S, D)).transpose(1, 2).contiguous()
    v = dev_bf16(iid_normal_bf16(52, 2, B, Nkv, S, D)).transpose(1, 2).contiguous()
    want, _, _ = qb.attn_fwd(q, k, v, N, "BSND", scale=scale, return_stats=False)
    got = ulysses.ulysses_attention(q, k, v, ulysses.bsnd_attention(scale), comm_type=comm_type,
                                    heads_per_chunk=hpc)
    torch.cuda.synchronize()
    qb.check()
    assert torch.equal(got, want)
