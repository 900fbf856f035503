"""The MSA prefill pass and decode step as sequences of libmsa calls.

Buffers (outputs and zero-filled workspaces) are torch device tensors sized from
``msa_workspace_size``; allocation happens once in the ``*_buffers`` helpers, never inside a
step, so a step can be captured in a CUDA graph.
"""
from __future__ import annotations

import torch

from . import (BLOCK, INDEX_DIM, TOPK, OP_ATTN_DECODE, OP_ATTN_PREFILL, OP_ATTN_PREFILL_BACKWARD,
               OP_INDEX_SELECT_DECODE, msa_sparse_attn_prefill_backward,
               OP_INDEX_SELECT_PREFILL, Shape, msa_decode_step, msa_fp8_close_blocks, msa_fp8_quantize_blocks,
               msa_index_select, msa_index_select_chunk, msa_pool_index_keys, msa_pool_index_keys_chunk,
               msa_pooled_keys_append, msa_prefill_chunk_workspace_size,
               msa_sparse_attn_decode_fp8, msa_sparse_attn_prefill, msa_sparse_attn_prefill_chunk,
               msa_workspace_size)


def _ws(shape: Shape, op: int, n: int, device) -> torch.Tensor:
    size = msa_workspace_size(shape, op, n)
    if size == 0:
        raise ValueError(f"unsupported shape/op for workspace (op={op}, n={n})")
    return torch.zeros(size, dtype=torch.uint8, device=device)


def prefill_buffers(B: int, N: int, Hq: int, G: int, device, with_lse: bool = True, with_main: bool = True) -> dict:
    """Buffers of a prefill of N tokens; with_main=False leaves out the main branch's output and
    workspace (an index-branch-only run)."""
    shape = Shape.make(B, Hq, G)
    nb = max(1, N // BLOCK)
    return {
        "shape": shape, "N": N, "nb_cap": nb,
        "pooled": torch.zeros(B, G, nb, INDEX_DIM, dtype=torch.float32, device=device),
        "tail_sum": torch.zeros(B, G, INDEX_DIM, dtype=torch.float32, device=device),
        "sel": torch.empty(B, N, G, TOPK, dtype=torch.int32, device=device),
        "out": torch.empty(B, N, Hq, 128, dtype=torch.bfloat16, device=device) if with_main else None,
        "lse": torch.empty(B, N, Hq, dtype=torch.float32, device=device) if with_lse and with_main else None,
        "ws_select": _ws(shape, OP_INDEX_SELECT_PREFILL, N, device),
        "ws_attn": _ws(shape, OP_ATTN_PREFILL, N, device) if with_main else None,
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
    """One decode step: select, append the new token (KV + pooled keys), attend.
    ctx_len [B] int32 on the device = tokens cached before the step (the new token's position).
    Caches: k_cache/v_cache [B,G,l_cap,128] bf16, pooled [B,G,nb_cap,64] fp32, tail_sum [B,G,64].
    One msa_decode_step call: the selection comes first (it scores only blocks below the new
    token's own, which the append does not change), so the append runs in its shadow
    (programmatic dependent launch), and the attention, which needs both, waits for the
    append's completion (after the selection's).
    Returns (out [B,Hq,128], lse [B,Hq], sel [B,G,16])."""
    s, mp = bufs["shape"], bufs["max_pos"]
    msa_decode_step(s, q, q_idx, k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache, k_cache.shape[2], tail_sum,
                    pooled, pooled.shape[2], mp, bufs["sel"], bufs["out"], bufs["lse"], bufs["ws_select"],
                    bufs["ws_append"], bufs["ws_attn"], stream)
    return bufs["out"], bufs["lse"], bufs["sel"]


def fp8_cache(k_cache, v_cache, n_blocks_cap: int):
    """Empty FP8 cache matching bf16 caches [B, G, l_cap, 128]: codes (uint8, same layout) and
    per-block scales [B, G, n_blocks_cap] (fp32)."""
    B, G, l_cap, d = k_cache.shape
    dev = k_cache.device
    return {"k_codes": torch.zeros(B, G, l_cap, d, dtype=torch.uint8, device=dev),
            "v_codes": torch.zeros(B, G, l_cap, d, dtype=torch.uint8, device=dev),
            "k_scale": torch.ones(B, G, n_blocks_cap, dtype=torch.float32, device=dev),
            "v_scale": torch.ones(B, G, n_blocks_cap, dtype=torch.float32, device=dev),
            "nb_cap": n_blocks_cap}


def fp8_quantize_sequence(k_cache, v_cache, f8: dict, b: int, n_tokens: int, n_q_heads: int, stream=None):
    """Quantise the closed blocks of sequence b's first n_tokens positions (all groups)."""
    G, l_cap = k_cache.shape[1], k_cache.shape[2]
    msa_fp8_quantize_blocks(Shape.make(1, n_q_heads, G), k_cache[b], v_cache[b], l_cap, n_tokens,
                            f8["k_codes"][b], f8["v_codes"][b], f8["k_scale"][b], f8["v_scale"][b], f8["nb_cap"],
                            stream)


def decode_step_fp8(q, q_idx, k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache, tail_sum, pooled, f8: dict,
                    bufs: dict, stream=None):
    """One decode step over the FP8 cache: select, append the new token (bf16 cache + pooled
    keys), quantise the block it closes, attend (closed blocks from the e4m3 codes, the own
    block from bf16). Returns (out, lse, sel)."""
    s, mp = bufs["shape"], bufs["max_pos"]
    l_cap = k_cache.shape[2]
    nb_cap = pooled.shape[2]
    msa_index_select(s, q_idx, 1, ctx_len, mp, pooled, nb_cap, bufs["sel"], bufs["ws_select"], stream)
    msa_pooled_keys_append(s, k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache, l_cap, tail_sum, pooled,
                           nb_cap, bufs["ws_append"], stream)
    msa_fp8_close_blocks(s, ctx_len, k_cache, v_cache, l_cap, f8["k_codes"], f8["v_codes"], f8["k_scale"],
                         f8["v_scale"], f8["nb_cap"], bufs["ws_append"], stream)
    msa_sparse_attn_decode_fp8(s, q, f8["k_codes"], f8["v_codes"], f8["k_scale"], f8["v_scale"], f8["nb_cap"],
                               k_cache, v_cache, l_cap, ctx_len, mp, bufs["sel"], bufs["out"], bufs["lse"],
                               bufs["ws_attn"], stream)
    return bufs["out"], bufs["lse"], bufs["sel"]


def prefill_chunk(q, q_idx, k_idx, k_cache, v_cache, q_start: int, pooled, tail_sum, n_q_heads: int, stream=None,
                  with_lse: bool = True):
    """One chunk of a chunked prefill: the n tokens at positions q_start .. q_start + n - 1.
    q [B,n,Hq,128], q_idx/k_idx [B,n,G,64]; k_cache/v_cache [B,G,l_cap,128] must already hold the
    chunk's K and V rows; pooled [B,G,nb_cap,64] and tail_sum [B,G,64] hold the pooled state of
    positions 0 .. q_start - 1 and are advanced past the chunk. A convenience for tests and
    examples: it allocates the chunk's outputs and workspaces on every call (a serving loop
    would size them once). Returns (out, lse, sel, workspaces)."""
    B, n, G = q_idx.shape[0], q_idx.shape[1], q_idx.shape[2]
    dev = q.device
    shape = Shape.make(B, n_q_heads, G)
    nb_cap = pooled.shape[2]
    l_cap = k_cache.shape[2]
    sel = torch.empty(B, n, G, TOPK, dtype=torch.int32, device=dev)
    out = torch.empty(B, n, n_q_heads, 128, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, n, n_q_heads, dtype=torch.float32, device=dev) if with_lse else None
    ws_sel = torch.zeros(msa_workspace_size(shape, OP_INDEX_SELECT_PREFILL, q_start + n), dtype=torch.uint8, device=dev)
    ws = torch.zeros(msa_prefill_chunk_workspace_size(shape, q_start, n), dtype=torch.uint8, device=dev)
    msa_pool_index_keys_chunk(shape, k_idx, q_start, n, pooled, nb_cap, tail_sum, stream)
    msa_index_select_chunk(shape, q_idx, q_start, n, pooled, nb_cap, sel, ws_sel, stream)
    msa_sparse_attn_prefill_chunk(shape, q, k_cache, v_cache, l_cap, q_start, n, sel, out, lse, ws, stream)
    return out, lse, sel, {"ws_select": ws_sel, "ws_attn": ws}


def backward_buffers(B: int, N: int, Hq: int, G: int, device) -> dict:
    """Gradient outputs (fp32) and the zeroed workspace of the main branch's backward pass."""
    shape = Shape.make(B, Hq, G)
    return {"shape": shape, "N": N,
            "dq": torch.empty(B, N, Hq, 128, dtype=torch.float32, device=device),
            "dk": torch.empty(B, G, N, 128, dtype=torch.float32, device=device),
            "dv": torch.empty(B, G, N, 128, dtype=torch.float32, device=device),
            "ws": _ws(shape, OP_ATTN_PREFILL_BACKWARD, N, device)}


def prefill_backward(q, k, v, d_out, fwd: dict, bwd: dict, stream=None):
    """Backward pass of the main branch after a prefill whose buffers are `fwd` (sel, out, lse).
    Returns (dq, dk, dv)."""
    msa_sparse_attn_prefill_backward(bwd["shape"], q, k, v, bwd["N"], fwd["sel"], fwd["out"], fwd["lse"], d_out,
                                     bwd["dq"], bwd["dk"], bwd["dv"], bwd["ws"], stream)
    return bwd["dq"], bwd["dk"], bwd["dv"]
