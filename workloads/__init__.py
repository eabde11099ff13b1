"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This package holds input generation only: random draws, the bf16 storage cast of
the draws, the structured Q/K recipe and the random 128x128 block keep-masks.  It
contains none of the attention arithmetic (no scores, softmax, quantisation or
rounding of P); the oracle and the CUDA library each implement that on their own.
"""

from .gen import (  # noqa: F401
    CONFIGS,
    BLK,
    bf16_bits_from_f32,
    bf16_bits_to_f32,
    iid_normal_bf16,
    blocky_qk_bf16,
    block_keep_mask,
    sample_rows,
    random_atten_mask,
    random_pse_bf16,
    device_iid_normal_bf16,
    device_blocky_qk_bf16,
)
