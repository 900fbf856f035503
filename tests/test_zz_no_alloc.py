"""msa_index_select_decode_noalloc: the decode selection for callers that cannot allocate
device memory (an engine that owns all device memory through its own pool and allows no
allocation per step). It keeps its scratch in a fixed array inside libmsa. These checks call
it through the C ABI and compare it with msa_index_select (decode mode, caller workspace) on
the same inputs, for two different problems in a row and then the first one again, so that
state left in the shared array by one call cannot leak into the next.

This file is collected last on purpose (its name sorts after the other test files). The
check that problems larger than the fixed scratch are rejected before any launch needs no GPU
and lives with the host-only tests of the C ABI.
"""
import ctypes

import pytest
import torch

import block_sparse_gqa_branch_b200 as msa
from block_sparse_gqa_branch_b200 import Shape, pipeline

pytestmark = pytest.mark.gpu


def _problem(B, G, positions, seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    max_pos = max(positions)
    nb_cap = max_pos // 128 + 1
    pooled = torch.randn(B, G, nb_cap, 64, device="cuda", generator=gen) * 0.1
    q_idx = torch.randn(B, G, 64, device="cuda", generator=gen).to(torch.bfloat16)
    q_pos = torch.tensor(positions, dtype=torch.int32, device="cuda")
    return dict(shape=Shape.make(B, 8 * G, G), B=B, G=G, max_pos=max_pos, nb_cap=nb_cap, pooled=pooled,
                q_idx=q_idx, q_pos=q_pos)


def _with_workspace(p):
    bufs = pipeline.decode_buffers(p["B"], 8 * p["G"], p["G"], p["max_pos"], "cuda")
    msa.msa_index_select(p["shape"], p["q_idx"], 1, p["q_pos"], p["max_pos"], p["pooled"], p["nb_cap"],
                         bufs["sel"], bufs["ws_select"])
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(bufs["ws_select"])[0] == 0
    return bufs["sel"].clone()


def _no_alloc(p):
    sel = torch.zeros(p["B"], p["G"], 16, dtype=torch.int32, device="cuda")
    L = msa.load()
    st = L.msa_index_select_decode_noalloc(ctypes.byref(p["shape"]), p["q_idx"].data_ptr(),
                                           p["q_pos"].data_ptr(), p["max_pos"], p["pooled"].data_ptr(),
                                           p["nb_cap"], sel.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, msa.msa_status_string(st)
    torch.cuda.synchronize()
    return sel


def test_no_alloc_select_matches_workspace_select(cuda_ok):
    first = _problem(16, 8, [131072] * 8 + [131071, 130000, 4000, 2048, 2047, 129, 0, 99999], seed=1)
    second = _problem(4, 8, [1048576, 524288, 262144, 65536], seed=2)
    for p in (first, second, first):
        ref = _with_workspace(p)
        got = _no_alloc(p)
        # selection ids are integers: the two paths must agree exactly
        assert torch.equal(got, ref)
        assert (got[..., 0] >= 0).all()

