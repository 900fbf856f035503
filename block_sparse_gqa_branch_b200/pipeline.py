"""The MSA prefill pass and decode step as sequences of libmsa calls.

Buffers (outputs and zero-filled workspaces) are torch device tensors sized from
``msa_workspace_size``; allocation happens once in the ``*_buffers`` helpers, never inside a
step, so a step can be captured in a CUDA graph.
"""
from __future__ import annotations

import torch

from . import (BLOCK, INDEX_DIM, TOPK, OP_ATTN_DECODE, OP_ATTN_PREFILL, OP_INDEX_SELECT_DECODE,
               OP_INDEX_SELECT_PREFILL, Shape, msa_index_select, msa_pool_index_keys,
               msa_pooled_keys_append, msa_sparse_attn_decode, msa_sparse_attn_prefill,
               msa_workspace_size)


def _ws(shape: Shape, op: int, n: int, device) -> torch.Tensor:
    size = msa_workspace_size(shape, op, n)
    if size == 0:
        raise ValueError(f"unsupported shape/op for workspace (op={op}, n={n})")
    return torch.zeros(size, dtype=torch.uint8, device=device)


def prefill_buffers(B: int, N: int, Hq: int, G: int, device, with_lse: bool = True) -> dict:
    shape = Shape.make(B, Hq, G)
    nb = max(1, N // BLOCK)
    return {
        "shape": shape, "N": N, "nb_cap": nb,
        "pooled": torch.zeros(B, G, nb, INDEX_DIM, dtype=torch.float32, device=device),
        "tail_sum": torch.zeros(B, G, INDEX_DIM, dtype=torch.float32, device=device),
        "sel": torch.empty(B, N, G, TOPK, dtype=torch.int32, device=device),
        "out": torch.empty(B, N, Hq, 128, dtype=torch.bfloat16, device=device),
        "lse": torch.empty(B, N, Hq, dtype=torch.float32, device=device) if with_lse else None,
        "ws_select": _ws(shape, OP_INDEX_SELECT_PREFILL, N, device),
        "ws_attn": _ws(shape, OP_ATTN_PREFILL, N, device),
    }


def prefill_index(q_idx, k_idx, bufs: dict, stream=None):
    """Index Branch of a prefill: pooling, then scores + top-k. Returns sel."""
    s, N, nb = bufs["shape"], bufs["N"], bufs["nb_cap"]
    msa_pool_index_keys(s, k_idx, N, bufs["pooled"], nb, bufs["tail_sum"], stream)
    msa_index_select(s, q_idx, N, None, N - 1, bufs["pooled"], nb, bufs["sel"], bufs["ws_select"], stream)
    return bufs["sel"]


def prefill_main(q, k, v, bufs: dict, stream=None):
    """Main Branch of a prefill on bufs['sel']. Returns (out, lse)."""
    msa_sparse_attn_prefill(bufs["shape"], q, k, v, bufs["N"], bufs["sel"], bufs["out"], bufs["lse"],
                            bufs["ws_attn"], stream)
    return bufs["out"], bufs["lse"]


def prefill(q, k, v, q_idx, k_idx, bufs: dict, stream=None):
    """Whole MSA prefill. Returns (out, lse, sel)."""
    prefill_index(q_idx, k_idx, bufs, stream)
    out, lse = prefill_main(q, k, v, bufs, stream)
    return out, lse, bufs["sel"]


def decode_buffers(B: int, Hq: int, G: int, max_pos: int, device, with_lse: bool = True) -> dict:
    shape = Shape.make(B, Hq, G)
    return {
        "shape": shape, "max_pos": max_pos,
        "sel": torch.empty(B, G, TOPK, dtype=torch.int32, device=device),
        "out": torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=device),
        "lse": torch.empty(B, Hq, dtype=torch.float32, device=device) if with_lse else None,
        "ws_append": torch.zeros(256, dtype=torch.uint8, device=device),
        "ws_select": _ws(shape, OP_INDEX_SELECT_DECODE, max_pos, device),
        "ws_attn": _ws(shape, OP_ATTN_DECODE, max_pos, device),
    }


def decode_step(q, q_idx, k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache, tail_sum, pooled,
                bufs: dict, stream=None):
    """One decode step: append the new token (KV + pooled keys), select, attend.
    ctx_len [B] int32 on the device = tokens cached before the step (the new token's position).
    Caches: k_cache/v_cache [B,G,l_cap,128] bf16, pooled [B,G,nb_cap,64] fp32, tail_sum [B,G,64].
    Returns (out [B,Hq,128], lse [B,Hq], sel [B,G,16])."""
    s, mp = bufs["shape"], bufs["max_pos"]
    l_cap = k_cache.shape[2]
    nb_cap = pooled.shape[2]
    msa_pooled_keys_append(s, k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache, l_cap, tail_sum, pooled,
                           nb_cap, bufs["ws_append"], stream)
    msa_index_select(s, q_idx, 1, ctx_len, mp, pooled, nb_cap, bufs["sel"], bufs["ws_select"], stream)
    msa_sparse_attn_decode(s, q, k_cache, v_cache, l_cap, ctx_len, mp, bufs["sel"], bufs["out"], bufs["lse"],
                           bufs["ws_attn"], stream)
    return bufs["out"], bufs["lse"], bufs["sel"]
