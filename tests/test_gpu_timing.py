"""The library's per-kernel timing on the GPU: while switched on, every eager launch of a
prefill is recorded with its kernel id and a device time, in launch order; stream captures
are not timed; switched off, nothing is recorded."""
import pytest
import torch

import synth
from block_sparse_gqa_branch_b200 import msa_kernel_launches, msa_kernel_timing_enable, msa_kernel_timing_read, pipeline

pytestmark = pytest.mark.gpu


def test_prefill_launches_are_timed_in_order(cuda_ok):
    w = synth.small_workload(N=2500, Hq=16, G=2, B=1, seed=77)
    x = synth.prefill_inputs_torch(w, "cuda")
    bufs = pipeline.prefill_buffers(w.B, w.N, w.Hq, w.G, "cuda")
    pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], bufs)
    torch.cuda.synchronize()
    msa_kernel_timing_read()                                  # drop anything earlier
    l0 = msa_kernel_launches()
    assert msa_kernel_timing_enable(True) is False
    try:
        pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], bufs)
        torch.cuda.synchronize()
    finally:
        msa_kernel_timing_enable(False)
    recs = msa_kernel_timing_read()
    names = [n for n, _ in recs]
    assert len(recs) == msa_kernel_launches() - l0
    # pooling, split keys, selection, inverted index (count, scan, fill), attention, combine
    assert names == ["pool", "split_keys", "select_prefill", "inverted_index", "inverted_index", "inverted_index",
                     "attn_prefill", "combine"], names
    assert all(ms > 0.0 for _, ms in recs)
    assert msa_kernel_timing_read() == []                     # read once
    # off again: nothing recorded
    pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], bufs)
    torch.cuda.synchronize()
    assert msa_kernel_timing_read() == []


def test_captured_launches_are_not_timed(cuda_ok):
    a = torch.randn(64, 1024, device="cuda")
    idx = torch.empty(64, 15, dtype=torch.int32, device="cuda")
    from block_sparse_gqa_branch_b200 import msa_topk_rows
    msa_topk_rows(a, 15, idx)
    torch.cuda.synchronize()
    msa_kernel_timing_read()
    msa_kernel_timing_enable(True)
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            msa_topk_rows(a, 15, idx)
        g.replay()
        msa_topk_rows(a, 15, idx)                             # one eager launch
        torch.cuda.synchronize()
    finally:
        msa_kernel_timing_enable(False)
    recs = msa_kernel_timing_read()
    assert [n for n, _ in recs] == ["topk"]
    del g
