"""Block-mask estimation for block-sparse attention, a plain reading, in fp64.

TEST INFRASTRUCTURE ONLY (see the package header).

Source: EagleQBSA article ("昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,视频生成端到端加速1.6倍"),
section "背景介绍": EagleQBSA builds on the adaptive block-sparse attention feature
AdaBSA, which computes only the 128x128 blocks of the attention map that a block mask
selects; section "MindIE SD调用方式" passes that mask as block_sparse_mask with
block_shape=[128,128].  The article names the selector but does not describe it.

Reading (the plainest one consistent with the article; listed in the design notes):

1. Pool each 128-token block of Q and of K to its mean row (over the block's valid
   tokens only; a tail block averages fewer rows).
2. Score each (query block i, key block j) pair by scale * <q_mean_i, k_mean_j>, with key
   head h // (N_q / N_kv) for query head h.  This equals the mean of the scaled token
   scores scale * q_r . k_c over the block (bilinearity), i.e. the block's average logit.
3. Keep, per query block, the n_keep highest-scoring key blocks; equal scores go to the
   lower key-block index.  n_keep = max(1, min(n_kb, round(keep * n_kb))), the count rule
   of the synthetic masks of the workloads.  1 = compute the block.

Parity pins (tests): block means of constant and affine tensors; the block score equals
the block average of the dense token-score matrix computed directly from Q and K; top-k
against brute-force selection on small random scores, exact ties, keep = 1 (everything)
and n_keep = 1 (the argmax).
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64

BLOCK = 128


def block_means(x_bits: np.ndarray) -> np.ndarray:
    """bf16 bits [B, N, S, D] -> fp64 [B, N, ceil(S/128), D]: mean row of each 128-token block."""
    x = bf16_to_f64(x_bits)
    B, N, S, D = x.shape
    nb = -(-S // BLOCK)
    out = np.zeros((B, N, nb, D))
    for i in range(nb):
        r0, r1 = i * BLOCK, min(S, (i + 1) * BLOCK)
        out[:, :, i] = x[:, :, r0:r1].mean(axis=2)
    return out


def block_scores(q_mean: np.ndarray, k_mean: np.ndarray, scale: float) -> np.ndarray:
    """[B, Nq, nqb, D] x [B, Nkv, nkb, D] -> [B, Nq, nqb, nkb] = scale * q_mean . k_mean (GQA heads)."""
    B, Nq = q_mean.shape[:2]
    Nkv = k_mean.shape[1]
    group = Nq // Nkv
    out = np.empty((B, Nq, q_mean.shape[2], k_mean.shape[2]))
    for h in range(Nq):
        out[:, h] = scale * np.einsum("bid,bjd->bij", q_mean[:, h], k_mean[:, h // group])
    return out


def keep_count(n_kb: int, keep: float) -> int:
    return max(1, min(n_kb, int(round(keep * n_kb))))


def topk_mask(scores: np.ndarray, n_keep: int) -> np.ndarray:
    """uint8 mask of the n_keep largest scores along the last axis; ties to the lower index."""
    n_kb = scores.shape[-1]
    flat = scores.reshape(-1, n_kb)
    out = np.zeros(flat.shape, dtype=np.uint8)
    for r in range(flat.shape[0]):
        # descending score, then ascending index: a stable sort of the negated scores
        order = np.argsort(-flat[r], kind="stable")
        out[r, order[:n_keep]] = 1
    return out.reshape(scores.shape)


def estimate_block_mask(q_bits: np.ndarray, k_bits: np.ndarray, scale: float, keep: float):
    """Steps 1-3 above.  Returns (mask uint8 [B, Nq, nqb, nkb], scores fp64 of the same shape)."""
    qm = block_means(q_bits)
    km = block_means(k_bits)
    s = block_scores(qm, km, scale)
    return topk_mask(s, keep_count(s.shape[-1], keep)), s
