"""The C ABI without a GPU: the library loads, exports what include/msa.h declares, sizes
workspaces, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

import block_sparse_gqa_branch_b200 as msa
from block_sparse_gqa_branch_b200 import Shape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")

FAKE = 0x10000          # an aligned, never dereferenced address: validation fails before use
FAKE2 = 0x20000


@pytest.fixture(scope="module")
def L():
    from block_sparse_gqa_branch_b200 import build
    build.build()
    return msa.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert sorted(names) == sorted(msa.EXPORTED_SYMBOLS)


def test_version_and_status_strings(L):
    assert msa.msa_abi_version() == 1
    for code in range(7):
        assert msa.msa_status_string(code) not in ("", "unknown status")
    assert msa.msa_status_string(99) == "unknown status"


def test_workspace_sizes(L):
    s = Shape.make(16, 64, 8)
    assert msa.msa_workspace_size(s, msa.OP_ATTN_DECODE, 131072) >= 256 + 16 * 8 * 16 * 8 * 130 * 4
    assert msa.msa_workspace_size(s, msa.OP_INDEX_SELECT_DECODE, 131072) > 256
    # prefill selection: the header, then the fully-past blocks' pooled keys split into three bf16
    # terms (3 x 64 x 2 B per block and group), in whole 64-block chunks
    for n, nbp in ((1, 64), (128, 64), (129, 64), (4096, 64), (8193, 64), (8321, 128), (131072, 1024)):
        assert msa.msa_workspace_size(s, msa.OP_INDEX_SELECT_PREFILL, n) == 256 + 16 * 8 * 3 * nbp * 128, n
    assert msa.msa_workspace_size(s, msa.OP_INDEX_SELECT_PREFILL, 0) == 0
    assert msa.msa_workspace_size(s, 17, 10) == 0
    assert msa.msa_workspace_size(Shape.make(1, 6, 4), msa.OP_ATTN_DECODE, 10) == 0      # Hq % G
    assert msa.msa_workspace_size(Shape.make(1, 24, 1), msa.OP_ATTN_DECODE, 10) == 0     # Hg = 24
    assert msa.msa_workspace_size(Shape.make(1, 8, 1, head_dim=64), msa.OP_ATTN_DECODE, 10) == 0
    assert msa.msa_workspace_size(s, msa.OP_INDEX_SELECT_DECODE, 1 << 25) == 0          # beyond max


def test_selftest_validates_its_workspace(L):
    assert L.msa_selftest_wait_timeout(None, 256, None) == 3                 # MSA_ERR_WORKSPACE
    assert L.msa_selftest_wait_timeout(FAKE, 100, None) == 3                  # too small
    assert L.msa_selftest_wait_timeout(FAKE + 2, 256, None) == 3              # misaligned


def _shape(**kw):
    base = dict(batch=1, n_q_heads=8, n_kv_groups=1)
    base.update(kw)
    return Shape.make(**base)


def test_validation_errors_before_launch(L):
    s = _shape()
    bs = ctypes.byref(s)
    # null / misaligned pointers
    assert L.msa_pool_index_keys(bs, None, 256, FAKE, 2, None, None) == 1
    assert L.msa_pool_index_keys(bs, FAKE + 2, 256, FAKE, 2, None, None) == 1
    assert L.msa_pool_index_keys(bs, FAKE, 256, FAKE, 1, None, None) == 1            # nb_cap too small
    assert L.msa_pool_index_keys(None, FAKE, 256, FAKE, 2, None, None) == 1
    # unsupported constants
    for bad in (dict(head_dim=64), dict(index_dim=32), dict(block_size=64), dict(top_k=8)):
        assert L.msa_pool_index_keys(ctypes.byref(_shape(**bad)), FAKE, 256, FAKE, 2, None, None) == 2
    assert L.msa_pool_index_keys(ctypes.byref(_shape(n_q_heads=12, n_kv_groups=1)), FAKE, 256, FAKE, 2, None, None) == 2
    assert L.msa_pool_index_keys(ctypes.byref(_shape(n_q_heads=12, n_kv_groups=8)), FAKE, 256, FAKE, 2, None, None) == 1
    # select: workspace missing / too small; decode with n_queries != 1
    assert L.msa_index_select(bs, FAKE, 4096, None, 4095, FAKE, 32, FAKE2, None, 0, None) == 3
    assert L.msa_index_select(bs, FAKE, 4096, None, 4095, FAKE, 32, FAKE2, FAKE, 16, None) == 3
    assert L.msa_index_select(bs, FAKE, 2, FAKE, 4095, FAKE, 32, FAKE2, FAKE, 1 << 20, None) == 1
    assert L.msa_index_select(bs, FAKE, 1, FAKE, 1 << 26, FAKE, 1 << 20, FAKE2, FAKE, 1 << 30, None) == 2
    need = msa.msa_workspace_size(s, msa.OP_INDEX_SELECT_DECODE, 4095)
    assert L.msa_index_select(bs, FAKE, 1, FAKE, 4095, FAKE, 32, FAKE2, FAKE, need - 16, None) == 3
    assert L.msa_index_select(bs, FAKE, 1, FAKE, 4095, FAKE, 30, FAKE2, FAKE, need, None) == 1   # nb_cap
    # prefill attention
    assert L.msa_sparse_attn_prefill(bs, FAKE, FAKE, None, 100, FAKE, FAKE, None, FAKE, 1 << 20, None) == 1
    assert L.msa_sparse_attn_prefill(bs, FAKE, FAKE, FAKE, 0, FAKE, FAKE, None, FAKE, 1 << 20, None) == 1
    assert L.msa_sparse_attn_prefill(bs, FAKE, FAKE, FAKE, 100, FAKE, FAKE, FAKE + 2, FAKE, 1 << 20, None) == 1
    assert L.msa_sparse_attn_prefill(bs, FAKE, FAKE, FAKE, 100, FAKE, FAKE, None, None, 0, None) == 3
    # 32-bit device indices: B*N*Hq*16 partial rows must stay below 2^31 (here exactly 2^31)
    big = ctypes.byref(_shape(n_q_heads=64, n_kv_groups=8))
    assert L.msa_sparse_attn_prefill(big, FAKE, FAKE, FAKE, 1 << 21, FAKE, FAKE, None, FAKE, 1 << 62, None) == 2
    assert L.msa_sparse_attn_prefill(big, FAKE, FAKE, FAKE, 1 << 20, FAKE, FAKE, None, FAKE, 16, None) == 3
    # decode attention: position bound beyond the cache, workspace
    assert L.msa_sparse_attn_decode(bs, FAKE, FAKE, FAKE, 1000, FAKE, 1000, FAKE, FAKE, None, FAKE, 1 << 20, None) == 1
    assert L.msa_sparse_attn_decode(bs, FAKE, FAKE, FAKE, 1000, FAKE, 999, FAKE, FAKE, None, FAKE, 64, None) == 3
    # append: k_new without v_new
    assert L.msa_pooled_keys_append(bs, FAKE, FAKE, None, FAKE, FAKE, FAKE, 10, FAKE, FAKE, 1, FAKE, 256, None) == 1
    assert L.msa_pooled_keys_append(bs, FAKE, None, None, FAKE, None, None, 0, FAKE, FAKE, 1, FAKE, 16, None) == 3


def test_decode_step_validates_all_three_steps_before_launch(L):
    s = _shape(batch=2, n_q_heads=16, n_kv_groups=2)
    bs = ctypes.byref(s)
    max_pos, l_cap, nb_cap = 4095, 4096, 32     # every call below fails validation: nothing launches
    ws_sel = msa.msa_workspace_size(s, msa.OP_INDEX_SELECT_DECODE, max_pos)
    ws_att = msa.msa_workspace_size(s, msa.OP_ATTN_DECODE, max_pos)
    ok = [bs, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE2, FAKE, FAKE, l_cap, FAKE, FAKE, nb_cap, max_pos,
          FAKE2, FAKE, None, FAKE, ws_sel, FAKE, 256, FAKE, ws_att, None]

    def call(**kw):
        args = list(ok)
        names = ["shape", "q", "q_idx", "k_idx_new", "k_new", "v_new", "ctx_len", "k_cache", "v_cache", "l_cap",
                 "tail_sum", "pooled", "nb_cap", "max_pos", "sel", "out", "lse", "ws_select", "ws_select_bytes",
                 "ws_append", "ws_append_bytes", "ws_attn", "ws_attn_bytes", "stream"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return L.msa_decode_step(*args)

    assert call(shape=None) == 1
    assert call(k_new=None, v_new=None) == 1               # the step always appends K and V
    assert call(v_new=None) == 1
    assert call(q_idx=FAKE + 2) == 1                       # misaligned
    assert call(sel=None) == 1
    assert call(q=None) == 1
    assert call(ctx_len=None) == 1
    assert call(max_pos=l_cap) == 1                        # positions beyond the cache
    assert call(nb_cap=max_pos // 128 - 1) == 1             # too small for the last position
    assert call(max_pos=1 << 26, l_cap=1 << 27, nb_cap=1 << 20) == 2
    assert call(ws_select_bytes=ws_sel - 16) == 3
    assert call(ws_append=None) == 3
    assert call(ws_append_bytes=16) == 3
    assert call(ws_attn_bytes=ws_att - 256) == 3
    assert call(ws_attn=FAKE + 8) == 3                     # misaligned


def test_binding_rejects_host_tensors(L):
    import torch
    with pytest.raises(ValueError):
        msa.msa_pool_index_keys(_shape(), torch.zeros(1, 256, 1, 64, dtype=torch.bfloat16), 256,
                                torch.zeros(1, 1, 2, 64), 2)


def test_topk_validation_before_launch(L):
    ok = (FAKE, 100, 1024, 15, FAKE2, None, None)
    for bad in ((None,) + ok[1:],                       # null scores
                (FAKE + 4,) + ok[1:],                   # misaligned scores
                ok[:4] + (None,) + ok[5:],              # null idx
                ok[:4] + (FAKE2 + 8,) + ok[5:],         # misaligned idx
                ok[:5] + (FAKE + 2,) + ok[6:],          # misaligned val
                ok[:1] + (-1,) + ok[2:],                # rows < 0
                ok[:3] + (0,) + ok[4:], ok[:3] + (17,) + ok[4:],     # k outside 1..16
                ok[:2] + (14,) + ok[3:],                # n < k
                ok[:2] + ((1 << 30) + 4,) + ok[3:]):    # n too large
        assert L.msa_topk_rows(*bad) == 1, bad
    assert L.msa_topk_rows(None, 0, 1024, 15, None, None, None) == 0    # no rows: nothing to do


def test_no_alloc_select_rejects_problems_beyond_its_scratch(L):
    # msa_index_select_decode_noalloc keeps its scratch in a fixed 2 MiB device array; a
    # problem whose scratch would not fit returns MSA_ERR_WORKSPACE on the host, before any
    # CUDA call, so the fake pointers are never touched
    shape = ctypes.byref(Shape.make(64, 512, 64))
    max_pos = 4_000_000
    assert L.msa_index_select_decode_noalloc(shape, FAKE, FAKE2, max_pos, FAKE, max_pos // 128 + 1, FAKE,
                                             None) == 3
    # B * G = 272 fits at the largest supported position; B * G = 1024 only up to 2,228,351
    ok_shape = ctypes.byref(Shape.make(34, 8 * 8, 8))
    assert L.msa_index_select_decode_noalloc(ok_shape, FAKE, FAKE2, (1 << 24) - 1, FAKE, 1 << 17, FAKE + 2,
                                             None) == 1      # misaligned sel: rejected as an argument
    big = ctypes.byref(Shape.make(128, 8 * 8, 8))
    assert L.msa_index_select_decode_noalloc(big, FAKE, FAKE2, 2_228_352 + 128 * 1024 * 8, FAKE, 1 << 17, FAKE,
                                             None) == 3
    # invalid arguments come first
    assert L.msa_index_select_decode_noalloc(shape, None, FAKE2, 100, FAKE, 1, FAKE, None) == 1
    assert L.msa_index_select_decode_noalloc(shape, FAKE, FAKE2, 1 << 25, FAKE, 1 << 18, FAKE, None) == 2


def test_fp8_entry_points_validate_before_launch(L):
    s = ctypes.byref(_shape())
    # quantise: n_tokens beyond the cache, nb_cap too small, misaligned codes; zero blocks = nothing to do
    assert L.msa_fp8_quantize_blocks(s, FAKE, FAKE, 100, 200, FAKE, FAKE, FAKE, FAKE, 4, None) == 1
    assert L.msa_fp8_quantize_blocks(s, FAKE, FAKE, 1024, 1024, FAKE, FAKE, FAKE, FAKE, 7, None) == 1
    assert L.msa_fp8_quantize_blocks(s, FAKE, FAKE, 1024, 1024, FAKE + 8, FAKE, FAKE, FAKE, 8, None) == 1
    assert L.msa_fp8_quantize_blocks(s, FAKE, FAKE, 1024, 100, FAKE, FAKE, FAKE, FAKE, 8, None) == 0
    assert L.msa_fp8_quantize_blocks(ctypes.byref(_shape(head_dim=64)), FAKE, FAKE, 1024, 1024, FAKE, FAKE, FAKE,
                                     FAKE, 8, None) == 2
    # close: missing workspace, misaligned scale
    assert L.msa_fp8_close_blocks(s, FAKE, FAKE, FAKE, 1024, FAKE, FAKE, FAKE, FAKE, 8, None, 0, None) == 3
    assert L.msa_fp8_close_blocks(s, FAKE, FAKE, FAKE, 1024, FAKE, FAKE, FAKE + 2, FAKE, 8, FAKE, 256, None) == 1
    # decode attention: nb_cap below max_pos / 128, position beyond the cache, workspace
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 8, FAKE, FAKE, 1024, FAKE, 1000, FAKE, FAKE, None, FAKE, 1 << 20, None]
    assert L.msa_sparse_attn_decode_fp8(s, *args[:5], 6, *args[6:]) == 1
    assert L.msa_sparse_attn_decode_fp8(s, *args[:10], 1024, *args[11:]) == 1
    assert L.msa_sparse_attn_decode_fp8(s, *args[:15], 64, None) == 3
    assert L.msa_sparse_attn_decode_fp8(s, None, *args[1:]) == 1


def test_chunk_entry_points_validate_before_launch(L):
    s = ctypes.byref(_shape(n_q_heads=16, n_kv_groups=2))
    big = msa.msa_prefill_chunk_workspace_size(Shape.make(1, 16, 2), 1000, 500)
    assert big > msa.msa_prefill_chunk_workspace_size(Shape.make(1, 16, 2), 0, 500) > 256
    assert msa.msa_prefill_chunk_workspace_size(Shape.make(1, 16, 2), -1, 500) == 0
    assert msa.msa_prefill_chunk_workspace_size(Shape.make(1, 16, 2), 0, 0) == 0
    # a whole prefill is the chunk at P = 0 against a cache of exactly n rows
    assert msa.msa_prefill_chunk_workspace_size(Shape.make(1, 16, 2), 0, 777) == \
        msa.msa_workspace_size(Shape.make(1, 16, 2), msa.OP_ATTN_PREFILL, 777)
    # pooling: no tail buffer, nb_cap too small, completed blocks without pooled
    assert L.msa_pool_index_keys_chunk(s, FAKE, 100, 50, FAKE, 4, None, None) == 1
    assert L.msa_pool_index_keys_chunk(s, FAKE, 100, 600, FAKE, 4, FAKE, None) == 1
    assert L.msa_pool_index_keys_chunk(s, FAKE, 100, 200, None, 4, FAKE, None) == 1
    assert L.msa_pool_index_keys_chunk(s, FAKE, 100, 0, FAKE, 4, FAKE, None) == 1
    # selection: workspace, nb_cap
    assert L.msa_index_select_chunk(s, FAKE, 1000, 500, FAKE, 11, FAKE2, None, 0, None) == 3
    assert L.msa_index_select_chunk(s, FAKE, 1000, 500, FAKE, 10, FAKE2, FAKE, 256, None) == 1
    # the workspace covers the split keys of every block below P + n
    need = msa.msa_workspace_size(_shape(n_q_heads=16, n_kv_groups=2), msa.OP_INDEX_SELECT_PREFILL, 1500)
    assert need > 256
    assert L.msa_index_select_chunk(s, FAKE, 1000, 500, FAKE, 11, FAKE2, FAKE, need - 16, None) == 3
    assert L.msa_index_select_chunk(s, FAKE, 1000, 500, FAKE, 11, FAKE2, FAKE + 8, need, None) == 3
    # attention: the chunk must fit in the cache; the workspace depends on P
    assert L.msa_sparse_attn_prefill_chunk(s, FAKE, FAKE, FAKE, 1400, 1000, 500, FAKE, FAKE, None, FAKE, big,
                                           None) == 1
    assert L.msa_sparse_attn_prefill_chunk(s, FAKE, FAKE, FAKE, 1500, 1000, 500, FAKE, FAKE, None, FAKE, big - 16,
                                           None) == 3


def test_kernel_timing_switch_and_empty_read(L):
    # no kernel is enqueued here: switching timing on and off and reading no records needs no GPU
    assert L.msa_kernel_timing_enable(1) == 0
    assert L.msa_kernel_timing_enable(1) == 1
    assert L.msa_kernel_timing_enable(0) == 1
    assert L.msa_kernel_timing_read(None, None, 0) == 0
    assert msa.msa_kernel_timing_read() == []
    assert set(msa.KERNEL_NAMES) == set(range(1, 15))
