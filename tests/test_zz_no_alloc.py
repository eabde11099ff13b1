"""qbsa_quantize_v_noalloc, the V quantiser for callers that cannot allocate device memory
during the call (code inside a custom allocator or pool callback, processes that reserve the
whole device heap up front, runtimes that forbid allocation on their streams).  It keeps its
scratch in a fixed array of the library instead of allocating it, and must give exactly the
codes and scales of qbsa_quantize_v.

The file is named so that pytest collects it after every other test file."""

import ctypes

import numpy as np
import pytest
import torch

import quantized_block_sparse_attn_b200 as qb
from workloads import iid_normal_bf16
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_quantize_v_noalloc_matches_allocating_entry_point():
    L = qb.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B, N, S, D = 2, 3, 3000, 128      # 12 chunks of 256 rows per head, ragged last chunk
    v = iid_normal_bf16(61, 2, B, N, S, D)
    v[1, 2, :, 9] = 0                  # an all-zero channel takes scale 1
    tv = dev_bf16(v)
    want_codes, want_scales = qb.quantize_v(tv)    # the allocating entry point
    qb.check()
    for _ in range(2):                 # two calls in a row: the shared scratch is cleared every call
        codes = torch.full((B, N, S, D), 0xAB, dtype=torch.uint8, device="cuda")
        scales = torch.full((B, N, D), -1.0, dtype=torch.float32, device="cuda")
        st = L.qbsa_quantize_v_noalloc(_p(tv), B, N, S, D, _p(codes), _p(scales), stream)
        assert st == 0, L.qbsa_last_error().decode()
        qb.check()
        assert torch.equal(codes, want_codes)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), want_scales.cpu().numpy().view(np.uint32))


def test_quantize_v_noalloc_rejects_sizes_beyond_its_scratch():
    """B*N*D words above the fixed 65536 is refused before anything is queued."""
    L = qb.lib()
    v = torch.zeros((1, 8, 128, 128), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros((1, 8, 128, 128), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((1, 8, 128), dtype=torch.float32, device="cuda")
    st = L.qbsa_quantize_v_noalloc(_p(v), 1, 600, 128, 128, _p(codes), _p(scales), None)
    assert st == 2
    assert b"qbsa_quantize_v" in L.qbsa_last_error()
