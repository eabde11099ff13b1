"""Ulysses sequence-parallel attention across ranks, with head-chunked communication.

FA_Power_Cap guide (Wan inference, Ulysses sequence parallelism; sections on the three
comm_type modes and the "comm_type=1 insertcomm" / "comm_type=2 blockattn" steps):

* Every rank holds a slice of the sequence of Q, K and V in BSND layout [B, S/P, N, D].
* comm_type 0 (baseline): one all-to-all per tensor scatters the heads and gathers the
  sequence ([B, S, N/P, D] per rank), attention runs on the local heads, and one
  all-to-all brings the output back to sequence slices.
* comm_type 1 (insert communication): the heads are split into chunks; chunk c's
  all-to-all -> attention -> all-to-all runs while the next chunk's all-to-all is in
  flight, so communication overlaps attention.
* comm_type 2 (block attention): as 1, and the local query sequence of each chunk is cut
  into 2 blocks that each attend to the full K / V of the chunk.

Heads of a chunk: with P ranks and `heads_per_chunk` local heads per chunk, chunk c holds
global heads [c * heads_per_chunk * P, (c + 1) * heads_per_chunk * P) (the guide splits the
head axis into chunks of heads_per_chunk * world_size), and after the all-to-all rank r
owns heads_per_chunk of them; K and V (GQA: fewer heads) are chunked in proportion.

The attention itself is a callable attn(q, k, v) -> out on [B, S, n, D] BSND tensors
(for instance ``bsnd_attention`` below, which runs this library's attn_fwd kernel).  On
GPUs the collectives are NCCL all_to_all_single calls; communication of chunk c + 1 is
issued on a side stream before chunk c's attention so the two overlap.  Nothing here
moves data through the host.
"""

from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def heads_to_sequence(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, S/P, N, D] sequence slice -> [B, S, N/P, D]: rank r receives heads
    [r N/P, (r + 1) N/P) of every rank's slice, laid out in rank (= sequence) order."""
    world = dist.get_world_size(group)
    B, S_loc, N, D = x.shape
    if N % world != 0:
        raise ValueError(f"{N} heads are not divisible by {world} ranks")
    n = N // world
    send = x.reshape(B, S_loc, world, n, D).permute(2, 0, 1, 3, 4).contiguous()  # [P, B, S/P, n, D]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)  # recv[s] = rank s's slice, my heads
    return recv.permute(1, 0, 2, 3, 4).reshape(B, world * S_loc, n, D)


def sequence_to_heads(y: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of heads_to_sequence: [B, S, N/P, D] -> [B, S/P, N, D] (rank r keeps sequence
    slice r of every rank's heads, laid out in rank (= head) order)."""
    world = dist.get_world_size(group)
    B, S, n, D = y.shape
    if S % world != 0:
        raise ValueError(f"sequence {S} is not divisible by {world} ranks")
    S_loc = S // world
    send = y.reshape(B, world, S_loc, n, D).permute(1, 0, 2, 3, 4).contiguous()  # [P, B, S/P, n, D]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)  # recv[s] = my sequence slice of rank s's heads
    return recv.permute(1, 2, 0, 3, 4).reshape(B, S_loc, world * n, D)


def _chunk_attention(q, k, v, attn, block_count: int):
    if block_count == 1:
        return attn(q, k, v)
    blocks = torch.tensor_split(q, block_count, dim=1)
    return torch.cat([attn(qb, k, v) for qb in blocks], dim=1)


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, attn: Callable, *, comm_type: int = 0,
                      heads_per_chunk: Optional[int] = None, group=None) -> torch.Tensor:
    """Attention of sequence-sliced BSND inputs on every rank: q [B, S/P, N, D], k and v
    [B, S/P, N_kv, D] (N_kv dividing N); returns this rank's output slice [B, S/P, N, D].
    comm_type 0 / 1 / 2 as in the module docstring; heads_per_chunk (local query heads per
    chunk, comm_type 1 and 2) must divide N / P, and each chunk's K / V share must be whole heads."""
    world = dist.get_world_size(group)
    N, Nkv = q.shape[2], k.shape[2]
    if N % world != 0 or Nkv % world != 0 or N % Nkv != 0:
        raise ValueError(f"heads N={N}, N_kv={Nkv} must be divisible by {world} ranks and N by N_kv")
    if comm_type == 0:
        qg, kg, vg = (heads_to_sequence(t, group) for t in (q, k, v))
        return sequence_to_heads(attn(qg, kg, vg), group)
    if comm_type not in (1, 2):
        raise ValueError("comm_type must be 0, 1 or 2")
    local_heads = N // world
    hpc = heads_per_chunk or local_heads
    ratio = N // Nkv
    if local_heads % hpc != 0 or hpc % ratio != 0:
        raise ValueError(f"heads_per_chunk {hpc} must divide the {local_heads} local heads and be a multiple of {ratio}")
    n_chunks = local_heads // hpc
    wq, wk = hpc * world, hpc * world // ratio
    block_count = 2 if comm_type == 2 else 1
    chunks = [(q[:, :, c * wq:(c + 1) * wq], k[:, :, c * wk:(c + 1) * wk], v[:, :, c * wk:(c + 1) * wk])
              for c in range(n_chunks)]

    use_streams = q.is_cuda
    comm = torch.cuda.Stream(device=q.device) if use_streams else None
    main = torch.cuda.current_stream(q.device) if use_streams else None

    def exchange(c):
        if not use_streams:
            return tuple(heads_to_sequence(t, group) for t in chunks[c])
        comm.wait_stream(main)
        with torch.cuda.stream(comm):
            return tuple(heads_to_sequence(t, group) for t in chunks[c])

    outs = []
    pending = exchange(0)
    for c in range(n_chunks):
        if use_streams:
            main.wait_stream(comm)
            for t in pending:
                t.record_stream(main)
        cur = pending
        if c + 1 < n_chunks:
            pending = exchange(c + 1)  # the next chunk's exchange overlaps this chunk's attention
        outs.append(sequence_to_heads(_chunk_attention(*cur, attn, block_count), group))
    return torch.cat(outs, dim=2)


def bsnd_attention(scale: float, **kwargs) -> Callable:
    """attn(q, k, v) on bf16 BSND CUDA tensors through this library's attn_fwd kernel."""
    from ._binding import attn_fwd

    def attn(q, k, v):
        out, _, _ = attn_fwd(q.contiguous(), k.contiguous(), v.contiguous(), q.shape[2], "BSND", scale=scale,
                             return_stats=False, **kwargs)
        return out

    return attn
