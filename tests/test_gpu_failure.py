"""Failure detection on the GPU without a fault: a kernel whose only wait can never complete
must give up after its bounded wait, record MSA_ERR_TIMEOUT in the workspace, and leave the
context usable for the next launches."""
import time

import numpy as np
import pytest
import torch

import synth
from block_sparse_gqa_branch_b200 import (Shape, msa_get_device_status, msa_pool_index_keys,
                                          msa_selftest_wait_timeout)
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives(cuda_ok):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    msa_selftest_wait_timeout(ws)
    st, info = msa_get_device_status(ws)          # synchronises the stream
    elapsed = time.time() - t0
    assert st == 5, (st, info)                    # MSA_ERR_TIMEOUT
    assert info[0] == 9                           # the self-test kernel's id
    assert elapsed < 30.0                         # the wait gave up (about 2 s of SM clocks)
    assert msa_get_device_status(ws)[0] == 0      # cleared after reading
    # the context still runs kernels: pooling of one block matches the block mean
    k_idx = synth.normal_bf16(3, synth.STREAM_KI, (1, 128, 1, 64))
    pooled = torch.zeros(1, 1, 2, 64, device="cuda")
    msa_pool_index_keys(Shape.make(1, 4, 1), dev_bf16(k_idx), 128, pooled, 2, None)
    torch.cuda.synchronize()
    ref = synth.bf16_bits_to_f32(k_idx).astype(np.float64).mean(axis=1)[0, 0]
    np.testing.assert_allclose(pooled[0, 0, 0].cpu().numpy(), ref, rtol=1e-5, atol=1e-6)
