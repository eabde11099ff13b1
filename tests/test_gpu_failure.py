"""Failure detection on the GPU without a fault: a bounded wait on a barrier phase that nothing
completes must time out, be reported once by qbsa_check, and leave the context usable."""

import time

import numpy as np
import pytest
import torch

import quantized_block_sparse_attn_b200 as qb
from quantized_block_sparse_attn_b200._binding import _stream
from oracle import estimate
from workloads import iid_normal_bf16
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    L = qb.lib()
    dev = torch.device("cuda:0")
    assert L.qbsa_check(_stream(dev)) == 0  # nothing pending
    t0 = time.perf_counter()
    assert L.qbsa_wait_selftest(_stream(dev)) == 0
    status = L.qbsa_check(_stream(dev))
    waited = time.perf_counter() - t0
    assert status == 4, f"expected QBSA_ERR_TIMEOUT, got {status}"
    assert b"time limit" in L.qbsa_last_error()
    assert 1.5 <= waited <= 30.0          # the 2 s wait limit, not an endless loop
    assert L.qbsa_check(_stream(dev)) == 0  # the error word was cleared
    # the context still runs kernels and gets them right
    x = iid_normal_bf16(61, 0, 1, 2, 300, 128)
    got = qb.block_mean(dev_bf16(x)).cpu().numpy().astype(np.float64)
    assert np.abs(got - estimate.block_means(x)).max() <= 4e-5
    qb.check()
