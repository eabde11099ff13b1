"""B200 (sm_100a) fused attention forward: dense bf16 and quantized block-sparse (EagleQBSA).

The compute path is libqbsa.so (hand-written tcgen05 / TMA / TMEM kernels behind a C
ABI, declared in include/qbsa.h); this package is its thin ctypes binding.
"""

from ._binding import (  # noqa: F401
    INF_TOKENS,
    LIB_PATH,
    QbsaError,
    attn_fwd,
    attn_tile_schedule,
    block_mean,
    block_topk,
    bsa_fwd,
    block_lists,
    estimate_block_mask,
    check,
    lib,
    qbsa_fwd,
    quantize_qk,
    quantize_v,
)

from . import ulysses  # noqa: F401,E402  (sequence-parallel wrapper over torch.distributed)
