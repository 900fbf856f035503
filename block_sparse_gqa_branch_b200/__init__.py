"""MiniMax Sparse Attention (MSA) over GQA on B200 -- Python binding of libmsa.

This module only marshals arguments: torch device tensors become raw pointers, the current
torch stream becomes the CUDA stream, and every call goes to the C ABI declared in
``include/msa.h``. Every step of the computation runs in libmsa's CUDA kernels; there is no
CPU or PyTorch fallback, and using a function without the built library raises.

Function names match the C entry points. Tensors use the layouts of ``include/msa.h``:
q [B,N,Hq,128], k/v [B,G,N,128], q_idx/k_idx [B,N,G,64] (bf16), pooled [B,G,nb_cap,64]
(fp32), sel [B,N,G,16] (int32), out [B,N,Hq,128] (bf16).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "MSAError", "Shape", "load", "lib_path",
    "msa_abi_version", "msa_status_string", "msa_workspace_size",
    "msa_pool_index_keys", "msa_index_select", "msa_sparse_attn_prefill",
    "msa_pooled_keys_append", "msa_sparse_attn_decode", "msa_decode_step", "msa_get_device_status",
    "msa_index_select_decode_noalloc", "msa_selftest_wait_timeout", "msa_kernel_launches",
    "msa_topk_rows", "msa_fp8_quantize_blocks", "msa_fp8_close_blocks", "msa_sparse_attn_decode_fp8",
    "msa_pool_index_keys_chunk", "msa_index_select_chunk", "msa_sparse_attn_prefill_chunk",
    "msa_prefill_chunk_workspace_size", "msa_sparse_attn_prefill_backward",
    "msa_kernel_timing_enable", "msa_kernel_timing_read", "KERNEL_NAMES",
    "OP_INDEX_SELECT_PREFILL", "OP_ATTN_PREFILL_BACKWARD", "OP_INDEX_SELECT_DECODE", "OP_ATTN_PREFILL", "OP_ATTN_DECODE",
    "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libmsa.so")

OP_INDEX_SELECT_PREFILL, OP_INDEX_SELECT_DECODE, OP_ATTN_PREFILL, OP_ATTN_DECODE = 0, 1, 2, 3
OP_ATTN_PREFILL_BACKWARD = 4
HEAD_DIM, INDEX_DIM, BLOCK, TOPK = 128, 64, 128, 16

STATUS_NAMES = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARGUMENT", 2: "MSA_ERR_UNSUPPORTED",
                3: "MSA_ERR_WORKSPACE", 4: "MSA_ERR_CUDA", 5: "MSA_ERR_TIMEOUT",
                6: "MSA_ERR_DEVICE_BOUNDS"}

EXPORTED_SYMBOLS = [
    "msa_abi_version", "msa_status_string", "msa_last_cuda_error", "msa_kernel_launches",
    "msa_workspace_size",
    "msa_pool_index_keys", "msa_index_select", "msa_sparse_attn_prefill",
    "msa_pooled_keys_append", "msa_sparse_attn_decode", "msa_decode_step", "msa_get_device_status",
    "msa_index_select_decode_noalloc", "msa_selftest_wait_timeout", "msa_topk_rows",
    "msa_fp8_quantize_blocks", "msa_fp8_close_blocks", "msa_sparse_attn_decode_fp8",
    "msa_pool_index_keys_chunk", "msa_index_select_chunk", "msa_sparse_attn_prefill_chunk",
    "msa_prefill_chunk_workspace_size", "msa_sparse_attn_prefill_backward",
    "msa_kernel_timing_enable", "msa_kernel_timing_read",
]

# MSA_KERNEL_* ids of include/msa.h
KERNEL_NAMES = {1: "pool", 2: "select_prefill", 3: "select_decode", 4: "append", 5: "attn_decode",
                6: "attn_prefill", 7: "inverted_index", 8: "combine", 9: "selftest", 10: "fp8_quantize",
                11: "split_keys", 12: "attn_backward", 13: "backward_dot", 14: "topk"}


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_groups", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("index_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("top_k", ctypes.c_int32)]

    @classmethod
    def make(cls, batch: int, n_q_heads: int, n_kv_groups: int, head_dim: int = HEAD_DIM,
             index_dim: int = INDEX_DIM, block_size: int = BLOCK, top_k: int = TOPK) -> "Shape":
        return cls(batch, n_q_heads, n_kv_groups, head_dim, index_dim, block_size, top_k)


class MSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        extra = ""
        if status == 4 and _lib is not None:
            extra = " (cuda error %d)" % _lib.msa_last_cuda_error()
        super().__init__(f"{where}: {name}{extra}")


_lib = None
P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
SP = ctypes.POINTER(Shape)


def load():
    """Load libmsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(f"libmsa.so is not built ({lib_path}); run "
                               "python -m block_sparse_gqa_branch_b200.build")
        L = ctypes.CDLL(lib_path)
        L.msa_abi_version.restype = I32
        L.msa_status_string.restype = ctypes.c_char_p
        L.msa_status_string.argtypes = [ctypes.c_int]
        L.msa_last_cuda_error.restype = I32
        L.msa_kernel_launches.restype = ctypes.c_uint64
        L.msa_kernel_timing_enable.restype = I32
        L.msa_kernel_timing_enable.argtypes = [I32]
        L.msa_kernel_timing_read.restype = I32
        L.msa_kernel_timing_read.argtypes = [P, P, I32]
        L.msa_workspace_size.restype = SZ
        L.msa_workspace_size.argtypes = [SP, I32, I64]
        L.msa_prefill_chunk_workspace_size.restype = SZ
        L.msa_prefill_chunk_workspace_size.argtypes = [SP, I64, I64]
        for name, args in {
            "msa_pool_index_keys": [SP, P, I64, P, I64, P, P],
            "msa_index_select": [SP, P, I64, P, I64, P, I64, P, P, SZ, P],
            "msa_sparse_attn_prefill": [SP, P, P, P, I64, P, P, P, P, SZ, P],
            "msa_pooled_keys_append": [SP, P, P, P, P, P, P, I64, P, P, I64, P, SZ, P],
            "msa_sparse_attn_decode": [SP, P, P, P, I64, P, I64, P, P, P, P, SZ, P],
            "msa_decode_step": [SP, P, P, P, P, P, P, P, P, I64, P, P, I64, I64, P, P, P, P, SZ, P, SZ, P, SZ, P],
            "msa_get_device_status": [P, P, P],
            "msa_index_select_decode_noalloc": [SP, P, P, I64, P, I64, P, P],
            "msa_selftest_wait_timeout": [P, SZ, P],
            "msa_topk_rows": [P, I64, I64, I32, P, P, P],
            "msa_fp8_quantize_blocks": [SP, P, P, I64, I64, P, P, P, P, I64, P],
            "msa_fp8_close_blocks": [SP, P, P, P, I64, P, P, P, P, I64, P, SZ, P],
            "msa_sparse_attn_decode_fp8": [SP, P, P, P, P, P, I64, P, P, I64, P, I64, P, P, P, P, SZ, P],
            "msa_pool_index_keys_chunk": [SP, P, I64, I64, P, I64, P, P],
            "msa_index_select_chunk": [SP, P, I64, I64, P, I64, P, P, SZ, P],
            "msa_sparse_attn_prefill_chunk": [SP, P, P, P, I64, I64, I64, P, P, P, P, SZ, P],
            "msa_sparse_attn_prefill_backward": [SP, P, P, P, I64, P, P, P, P, P, P, P, P, SZ, P],
        }.items():
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libmsa takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libmsa takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise MSAError(status, where)


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


# ------------------------------------------------------------------------ the C entry points
def msa_abi_version() -> int:
    return load().msa_abi_version()


def msa_status_string(status: int) -> str:
    return load().msa_status_string(status).decode()


def msa_kernel_launches() -> int:
    return load().msa_kernel_launches()


def msa_kernel_timing_enable(on: bool) -> bool:
    """Switch per-kernel event timing on or off; returns the previous setting."""
    return bool(load().msa_kernel_timing_enable(1 if on else 0))


def msa_kernel_timing_read(cap: int = 1 << 16) -> list:
    """The timed launches since the last read, in launch order: [(kernel name, ms), ...]."""
    kid = (ctypes.c_int32 * cap)()
    ms = (ctypes.c_float * cap)()
    n = load().msa_kernel_timing_read(ctypes.cast(kid, ctypes.c_void_p), ctypes.cast(ms, ctypes.c_void_p), cap)
    if n < 0:
        raise MSAError(4, "msa_kernel_timing_read")
    return [(KERNEL_NAMES.get(int(kid[i]), str(int(kid[i]))), float(ms[i])) for i in range(n)]


def msa_workspace_size(shape: Shape, op: int, n: int) -> int:
    return load().msa_workspace_size(ctypes.byref(shape), op, n)


def msa_pool_index_keys(shape: Shape, k_idx, n_tokens: int, pooled, nb_cap: int, tail_sum=None,
                        stream=None):
    _check(load().msa_pool_index_keys(ctypes.byref(shape), _ptr(k_idx), n_tokens, _ptr(pooled),
                                      nb_cap, _ptr(tail_sum), _stream(stream)),
           "msa_pool_index_keys")


def msa_index_select(shape: Shape, q_idx, n_queries: int, q_pos, max_pos: int, pooled, nb_cap: int,
                     sel, workspace, stream=None):
    _check(load().msa_index_select(ctypes.byref(shape), _ptr(q_idx), n_queries, _ptr(q_pos), max_pos,
                                   _ptr(pooled), nb_cap, _ptr(sel), _ptr(workspace),
                                   _nbytes(workspace), _stream(stream)),
           "msa_index_select")


def msa_sparse_attn_prefill(shape: Shape, q, k, v, n_tokens: int, sel, out, lse, workspace,
                            stream=None):
    _check(load().msa_sparse_attn_prefill(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), n_tokens,
                                          _ptr(sel), _ptr(out), _ptr(lse), _ptr(workspace),
                                          _nbytes(workspace), _stream(stream)),
           "msa_sparse_attn_prefill")


def msa_pooled_keys_append(shape: Shape, k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache,
                           l_cap: int, tail_sum, pooled, nb_cap: int, workspace, stream=None):
    _check(load().msa_pooled_keys_append(ctypes.byref(shape), _ptr(k_idx_new), _ptr(k_new),
                                         _ptr(v_new), _ptr(ctx_len), _ptr(k_cache), _ptr(v_cache),
                                         l_cap, _ptr(tail_sum), _ptr(pooled), nb_cap,
                                         _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "msa_pooled_keys_append")


def msa_sparse_attn_decode(shape: Shape, q, k_cache, v_cache, l_cap: int, q_pos, max_pos: int, sel,
                           out, lse, workspace, stream=None):
    _check(load().msa_sparse_attn_decode(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                         l_cap, _ptr(q_pos), max_pos, _ptr(sel), _ptr(out), _ptr(lse),
                                         _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "msa_sparse_attn_decode")


def msa_decode_step(shape: Shape, q, q_idx, k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache, l_cap: int,
                    tail_sum, pooled, nb_cap: int, max_pos: int, sel, out, lse, ws_select, ws_append, ws_attn,
                    stream=None):
    _check(load().msa_decode_step(ctypes.byref(shape), _ptr(q), _ptr(q_idx), _ptr(k_idx_new), _ptr(k_new),
                                  _ptr(v_new), _ptr(ctx_len), _ptr(k_cache), _ptr(v_cache), l_cap, _ptr(tail_sum),
                                  _ptr(pooled), nb_cap, max_pos, _ptr(sel), _ptr(out), _ptr(lse),
                                  _ptr(ws_select), _nbytes(ws_select), _ptr(ws_append), _nbytes(ws_append),
                                  _ptr(ws_attn), _nbytes(ws_attn), _stream(stream)),
           "msa_decode_step")


def msa_get_device_status(workspace, stream=None):
    """Returns (status, info[4]) recorded by the device in the workspace, and clears it."""
    info = (ctypes.c_int32 * 4)()
    st = load().msa_get_device_status(_ptr(workspace), ctypes.cast(info, ctypes.c_void_p),
                                      _stream(stream))
    return st, list(info)


def msa_selftest_wait_timeout(workspace, stream=None):
    """Runs the failure-path self-test (see include/msa.h): a wait that expires after about
    2 s and is recorded as MSA_ERR_TIMEOUT in `workspace` (>= 256 zeroed bytes)."""
    _check(load().msa_selftest_wait_timeout(_ptr(workspace), _nbytes(workspace), _stream(stream)),
           "msa_selftest_wait_timeout")


def msa_index_select_decode_noalloc(shape: Shape, q_idx, q_pos, max_pos: int, pooled, nb_cap: int, sel,
                                    stream=None):
    """Decode selection that allocates nothing: its scratch is a fixed 2 MiB device array
    inside libmsa (see include/msa.h). Same results as msa_index_select in decode mode."""
    _check(load().msa_index_select_decode_noalloc(ctypes.byref(shape), _ptr(q_idx), _ptr(q_pos), max_pos,
                                                  _ptr(pooled), nb_cap, _ptr(sel), _stream(stream)),
           "msa_index_select_decode_noalloc")


def msa_topk_rows(scores, k: int, idx, val=None, stream=None):
    """Exp-free top-k of every row of scores (fp32 [rows, n]) into idx (int32 [rows, k]) and,
    when given, val (fp32 [rows, k])."""
    if scores.dim() != 2:
        raise ValueError("msa_topk_rows takes scores of shape [rows, n]")
    rows, n = scores.shape
    _check(load().msa_topk_rows(_ptr(scores), rows, n, k, _ptr(idx), _ptr(val), _stream(stream)),
           "msa_topk_rows")


def msa_fp8_quantize_blocks(shape: Shape, k_cache, v_cache, l_cap: int, n_tokens: int, k_codes, v_codes, k_scale,
                            v_scale, nb_cap: int, stream=None):
    """e4m3 codes and per-block scales of blocks j < n_tokens / 128 of the bf16 caches."""
    _check(load().msa_fp8_quantize_blocks(ctypes.byref(shape), _ptr(k_cache), _ptr(v_cache), l_cap, n_tokens,
                                          _ptr(k_codes), _ptr(v_codes), _ptr(k_scale), _ptr(v_scale), nb_cap,
                                          _stream(stream)),
           "msa_fp8_quantize_blocks")


def msa_fp8_close_blocks(shape: Shape, ctx_len, k_cache, v_cache, l_cap: int, k_codes, v_codes, k_scale, v_scale,
                         nb_cap: int, workspace, stream=None):
    """Quantise the blocks that this decode step's new tokens complete (after the append)."""
    _check(load().msa_fp8_close_blocks(ctypes.byref(shape), _ptr(ctx_len), _ptr(k_cache), _ptr(v_cache), l_cap,
                                       _ptr(k_codes), _ptr(v_codes), _ptr(k_scale), _ptr(v_scale), nb_cap,
                                       _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "msa_fp8_close_blocks")


def msa_sparse_attn_decode_fp8(shape: Shape, q, k_codes, v_codes, k_scale, v_scale, nb_cap: int, k_cache, v_cache,
                               l_cap: int, q_pos, max_pos: int, sel, out, lse, workspace, stream=None):
    """Decode attention over the FP8 cache (closed blocks) and the bf16 cache (own block)."""
    _check(load().msa_sparse_attn_decode_fp8(ctypes.byref(shape), _ptr(q), _ptr(k_codes), _ptr(v_codes),
                                             _ptr(k_scale), _ptr(v_scale), nb_cap, _ptr(k_cache), _ptr(v_cache),
                                             l_cap, _ptr(q_pos), max_pos, _ptr(sel), _ptr(out), _ptr(lse),
                                             _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "msa_sparse_attn_decode_fp8")


def msa_prefill_chunk_workspace_size(shape: Shape, q_start: int, n_queries: int) -> int:
    return load().msa_prefill_chunk_workspace_size(ctypes.byref(shape), q_start, n_queries)


def msa_pool_index_keys_chunk(shape: Shape, k_idx, q_start: int, n: int, pooled, nb_cap: int, tail_sum, stream=None):
    """Pool the blocks a chunk of index keys completes; keep the open block's running sum."""
    _check(load().msa_pool_index_keys_chunk(ctypes.byref(shape), _ptr(k_idx), q_start, n, _ptr(pooled), nb_cap,
                                            _ptr(tail_sum), _stream(stream)),
           "msa_pool_index_keys_chunk")


def msa_index_select_chunk(shape: Shape, q_idx, q_start: int, n: int, pooled, nb_cap: int, sel, workspace,
                           stream=None):
    """Selection for the chunk's queries at positions q_start .. q_start + n - 1."""
    _check(load().msa_index_select_chunk(ctypes.byref(shape), _ptr(q_idx), q_start, n, _ptr(pooled), nb_cap,
                                         _ptr(sel), _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "msa_index_select_chunk")


def msa_sparse_attn_prefill_chunk(shape: Shape, q, k_cache, v_cache, l_cap: int, q_start: int, n: int, sel, out, lse,
                                  workspace, stream=None):
    """Main Branch for the chunk's queries against the caches (positions 0 .. q_start + n - 1)."""
    _check(load().msa_sparse_attn_prefill_chunk(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), l_cap,
                                                q_start, n, _ptr(sel), _ptr(out), _ptr(lse), _ptr(workspace),
                                                _nbytes(workspace), _stream(stream)),
           "msa_sparse_attn_prefill_chunk")


def msa_sparse_attn_prefill_backward(shape: Shape, q, k, v, n_tokens: int, sel, out, lse, d_out, dq, dk, dv,
                                     workspace, stream=None):
    """Gradients dq [B,N,Hq,128], dk, dv [B,G,N,128] (fp32) of the prefill's main branch for the
    upstream gradient d_out, the selection held fixed."""
    _check(load().msa_sparse_attn_prefill_backward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), n_tokens,
                                                   _ptr(sel), _ptr(out), _ptr(lse), _ptr(d_out), _ptr(dq),
                                                   _ptr(dk), _ptr(dv), _ptr(workspace), _nbytes(workspace),
                                                   _stream(stream)),
           "msa_sparse_attn_prefill_backward")
