"""Seeded input recipes for the five workloads of the fused attention forward.

Every draw comes from ``numpy.random.Generator(PCG64)`` keyed by
``SeedSequence((seed, tensor_id, b, h))`` so that any single (batch, head) slice of
a full-size input can be regenerated on its own: the full-size parity checks
rebuild only the sampled heads on the host, bit for bit equal to what the bench
and the GPU tests upload.

Draws are made in float32 and stored as bf16 (round to nearest even), the storage
type of the dense path.  Nothing here computes attention.

Workload shapes follow the EagleQBSA article (昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,
section "EagleQBSA单算子性能验证分析", Fig 4.1: B=1, N=40, D=128, S from 8K to 128K;
section "文生视频任务评测": 1280x720, 65 frames, about 60k self-attention tokens) and
the npu_fusion_attention guide (昇腾 NPU 融合注意力算子详解与迁移指南, §4.1-§4.3:
BNSD / TND layouts, causal sparse modes, cumulative varlen lengths, GQA).
"""

from __future__ import annotations

import numpy as np

BLK = 128  # the 128x128 block shape of the block-sparse mask and of the quantisation blocks

# Tensor ids used in the seed key, one per tensor role.
_Q, _K, _V, _MASK, _MU_Q, _MU_K, _PSE, _AMASK = range(8)

# The five workloads.  ``seed`` is the workload index.
CONFIGS = {
    "tiny": dict(seed=0, layout="BNSD", B=1, Nq=2, Nkv=2, S=256, D=64, scale=1.0 / 8.0,
                 sparse_mode=0, qk="iid"),
    "causal": dict(seed=1, layout="BNSD", B=2, Nq=16, Nkv=16, S=4096, D=128,
                   scale=128 ** -0.5, sparse_mode=3, qk="iid"),
    "gqa_varlen": dict(seed=2, layout="TND", Nq=32, Nkv=8, D=128, seqlens=(1024, 5000, 10360),
                       scale=128 ** -0.5, sparse_mode=3, qk="iid"),
    "video": dict(seed=3, layout="BNSD", B=1, Nq=40, Nkv=40, S=61440, D=128,
                  scale=128 ** -0.5, sparse_mode=0, qk="blocky"),
    "qbsa": dict(seed=4, layout="BNSD", B=1, Nq=40, Nkv=40, D=128, S_list=(8192, 16384, 32768, 65536, 131072),
                 keep_list=(0.1, 0.5), scale=128 ** -0.5, qk="blocky"),
}


def _rng(seed: int, tensor_id: int, b: int = 0, h: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence((seed, tensor_id, b, h))))


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Store float32 values as bf16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def iid_normal_bf16(seed: int, tensor_id: int, n_batch: int, n_head: int, rows: int, d: int,
                    heads=None) -> np.ndarray:
    """bf16 bits of iid N(0,1) draws, shape [n_batch, n_head, rows, d] (BNSD order).

    ``heads`` (optional list of (b, h)) limits generation to those slices; the others
    stay zero.  A slice's values do not depend on which other slices are generated.
    """
    out = np.zeros((n_batch, n_head, rows, d), dtype=np.uint16)
    sel = heads if heads is not None else [(b, h) for b in range(n_batch) for h in range(n_head)]
    for b, h in sel:
        out[b, h] = bf16_bits_from_f32(_rng(seed, tensor_id, b, h).standard_normal((rows, d), dtype=np.float32))
    return out


def blocky_qk_bf16(seed: int, which: str, n_batch: int, n_head: int, rows: int, d: int,
                   noise_std: float = 0.3, heads=None) -> np.ndarray:
    """bf16 bits of locally coherent Q or K, shape [n_batch, n_head, rows, d].

    Per (b, h, 128-token block) one mean vector mu ~ N(0, I_d) is drawn and every token
    of the block is mu + N(0, noise_std^2 I_d).  This stands in for the video-DiT
    activations whose Q/K values concentrate inside a sequence block (EagleQBSA article,
    section "EagleQBSA量化叠加稀疏方案设计"); no model activations are available.
    """
    tid, mid = (_Q, _MU_Q) if which == "q" else (_K, _MU_K)
    nblk = -(-rows // BLK)
    out = np.zeros((n_batch, n_head, rows, d), dtype=np.uint16)
    sel = heads if heads is not None else [(b, h) for b in range(n_batch) for h in range(n_head)]
    for b, h in sel:
        mu = _rng(seed, mid, b, h).standard_normal((nblk, 1, d), dtype=np.float32)
        eps = _rng(seed, tid, b, h).standard_normal((nblk, BLK, d), dtype=np.float32)
        x = (mu + np.float32(noise_std) * eps).reshape(nblk * BLK, d)[:rows]
        out[b, h] = bf16_bits_from_f32(x)
    return out


def block_keep_mask(seed: int, n_batch: int, n_head: int, n_qb: int, n_kb: int, keep: float) -> np.ndarray:
    """uint8 [n_batch, n_head, n_qb, n_kb] block mask, 1 = compute the 128x128 block.

    Each (b, h, q-block) row keeps exactly max(1, round(keep * n_kb)) blocks: the
    diagonal block (index q-block * n_kb // n_qb) plus the rest drawn uniformly
    without replacement.  Keep fractions 0.1 and 0.5 match the sparsities 0.9 and
    0.5 of the EagleQBSA article (section "EagleQBSA单算子性能验证分析").
    """
    n_keep = max(1, min(n_kb, int(round(keep * n_kb))))
    out = np.zeros((n_batch, n_head, n_qb, n_kb), dtype=np.uint8)
    for b in range(n_batch):
        for h in range(n_head):
            rng = _rng(seed, _MASK, b, h)
            keys = rng.random((n_qb, n_kb))
            diag = (np.arange(n_qb) * n_kb) // n_qb
            keys[np.arange(n_qb), diag] = -1.0  # the diagonal sorts first
            idx = np.argsort(keys, axis=1, kind="stable")[:, :n_keep]
            np.put_along_axis(out[b, h], idx, 1, axis=1)
    return out


def random_atten_mask(seed: int, shape, p_masked: float = 0.3) -> np.ndarray:
    """uint8 explicit mask (1 = masked) with iid Bernoulli(p_masked) entries."""
    return (_rng(seed, _AMASK).random(shape) < p_masked).astype(np.uint8)


def random_pse_bf16(seed: int, shape, std: float = 1.0) -> np.ndarray:
    """bf16 bits of an iid N(0, std^2) positional bias."""
    return bf16_bits_from_f32(np.float32(std) * _rng(seed, _PSE).standard_normal(shape, dtype=np.float32))


def sample_rows(seed: int, n_rows: int, n_q_blocks_per_head: int = 8):
    """Deterministic q-block indices to check at full size: first, last, and random others."""
    n_qb = -(-n_rows // BLK)
    rng = _rng(seed, 99)
    pick = {0, n_qb - 1}
    extra = rng.choice(n_qb, size=min(n_qb, n_q_blocks_per_head), replace=False)
    for e in extra:
        if len(pick) >= min(n_qb, n_q_blocks_per_head):
            break
        pick.add(int(e))
    return sorted(pick)


# --------------------------------------------------------------------------------------
# device-side generation (bench sizes): same recipes, torch's seeded CUDA generator
# --------------------------------------------------------------------------------------

def _torch_gen(seed: int, tensor_id: int, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence((seed, tensor_id)).generate_state(1, dtype=np.uint64)[0] >> 1))
    return g


def device_iid_normal_bf16(seed: int, tensor_id: int, shape, device):
    """bf16 tensor of iid N(0,1) draws made on the device (torch Philox generator)."""
    import torch
    g = _torch_gen(seed, tensor_id, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def device_blocky_qk_bf16(seed: int, which: str, n_batch: int, n_head: int, rows: int, d: int, device,
                          noise_std: float = 0.3):
    """Device-made version of ``blocky_qk_bf16`` (same recipe, different random stream)."""
    import torch
    tid, mid = (_Q, _MU_Q) if which == "q" else (_K, _MU_K)
    nblk = -(-rows // BLK)
    mu = torch.randn((n_batch, n_head, nblk, 1, d), generator=_torch_gen(seed, mid, device), device=device)
    x = torch.randn((n_batch, n_head, nblk, BLK, d), generator=_torch_gen(seed, tid, device), device=device)
    x.mul_(noise_std).add_(mu)
    return x.reshape(n_batch, n_head, nblk * BLK, d)[:, :, :rows].to(torch.bfloat16).contiguous()
