"""fp64 CPU oracle for MiniMax Sparse Attention (MSA) over GQA -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. It shares nothing with the CUDA library (``block_sparse_gqa_branch_b200``)
and the library never imports it. The arithmetic lives in ``msa_oracle.c``; this file only
builds it with gcc, marshals numpy arrays through ctypes, and loops over sequences and groups.

Parity status of each function (what pins it) is listed in the tests that exercise it:
``oracle_pool``, ``block_scores``, ``select`` and ``attend`` are pinned (tests/test_oracle_pins.py);
nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmsa_oracle.so")
_lib = None

P = ctypes.c_void_p
I64 = ctypes.c_int64
INT = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile msa_oracle.c with gcc (plain C, -O2, no fast-math) into libmsa_oracle.so."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        # MSA_ORACLE_LIB lets the mutation test load a deliberately broken copy of the oracle
        _lib = ctypes.CDLL(os.environ.get("MSA_ORACLE_LIB") or build())
        _lib.oracle_bf16_to_f64.restype = ctypes.c_double
        _lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        _lib.oracle_pool.argtypes = [P, I64, I64, I64, I64, I64, P, P]
        _lib.oracle_block_scores.argtypes = [P, P, I64, I64, P]
        _lib.oracle_select_from_scores.restype = I64
        _lib.oracle_select_from_scores.argtypes = [P, I64, I64, P, P]
        _lib.oracle_select_fullsort.restype = I64
        _lib.oracle_select_fullsort.argtypes = [P, I64, I64, P]
        _lib.oracle_topk_rows.argtypes = [P, I64, I64, I64, P]
        _lib.oracle_attend_row_grad.argtypes = [P, P, P, I64, I64, P, I64, I64, P, P, P, P]
        _lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        _lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        _lib.oracle_e4m3_from_f32.restype = ctypes.c_uint8
        _lib.oracle_e4m3_from_f32.argtypes = [ctypes.c_float]
        _lib.oracle_fp8_quantize_block.restype = ctypes.c_float
        _lib.oracle_fp8_quantize_block.argtypes = [P, I64, P]
        _lib.oracle_attend_row_fp8.restype = I64
        _lib.oracle_attend_row_fp8.argtypes = [P, P, P, P, P, P, P, I64, I64, P, I64, I64, P, P]
        _lib.oracle_attend_row.restype = I64
        _lib.oracle_attend_row.argtypes = [P, P, P, I64, I64, P, I64, I64, P, P]
        _lib.oracle_select_rows.argtypes = [I64, P, P, P, I64, I64, I64, INT, P, P, P]
        _lib.oracle_attend_rows.argtypes = [I64, P, P, I64, P, P, I64, P, I64, I64, INT, INT,
                                            P, P, P]
    return _lib


def default_threads() -> int:
    return os.cpu_count() or 1


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- thin wrappers
def pool(k_idx_seq: np.ndarray, Bk: int = 128, nb_cap: Optional[int] = None):
    """k_idx_seq: [N, G, dI] bf16 bits of one sequence -> (pooled [G, nb_cap, dI] f64,
    tail_sum [G, dI] f64)."""
    k = _c(k_idx_seq, np.uint16)
    N, G, dI = k.shape
    nb = N // Bk if nb_cap is None else nb_cap
    pooled = np.zeros((G, max(nb, 1), dI), np.float64)
    tail = np.zeros((G, dI), np.float64)
    lib().oracle_pool(_p(k), N, G, dI, Bk, max(nb, 1), _p(pooled), _p(tail))
    return pooled[:, :nb], tail


def block_scores(q_idx_row: np.ndarray, pooled_g: np.ndarray, n_cand: int) -> np.ndarray:
    q = _c(q_idx_row, np.uint16)
    pg = _c(pooled_g, np.float64)
    s = np.zeros(max(n_cand, 1), np.float64)
    lib().oracle_block_scores(_p(q), _p(pg), q.shape[-1], n_cand, _p(s))
    return s[:n_cand]


def select_from_scores(s: np.ndarray, c: int, topk: int = 16):
    s = _c(s, np.float64) if len(s) else np.zeros(1, np.float64)
    sel = np.zeros(topk, np.int32)
    kth = np.zeros(1, np.float64)
    n = lib().oracle_select_from_scores(_p(s), c, topk, _p(sel), _p(kth))
    return sel, int(n), float(kth[0])


def select_fullsort(s: np.ndarray, c: int, topk: int = 16):
    s = _c(s, np.float64) if len(s) else np.zeros(1, np.float64)
    sel = np.zeros(topk, np.int32)
    n = lib().oracle_select_fullsort(_p(s), c, topk, _p(sel))
    return sel, int(n)


def topk_rows(scores: np.ndarray, k: int) -> np.ndarray:
    """Exp-free top-k of every row of fp32 scores [rows, n]: int32 [rows, k], best first
    (score descending, column ascending; NaN above +inf; -0 == +0)."""
    s = _c(scores, np.float32)
    rows, n = s.shape
    if not 1 <= k <= n:
        raise ValueError("topk_rows needs 1 <= k <= n")
    idx = np.zeros((rows, k), np.int32)
    lib().oracle_topk_rows(_p(s), rows, n, k, _p(idx))
    return idx


def attend_grad(t: np.ndarray, q_rows: np.ndarray, K: np.ndarray, V: np.ndarray, sel: Optional[np.ndarray],
                dO: np.ndarray, Bk: int = 128, nthreads: Optional[int] = None):
    """Gradient of step 4 for queries of one (sequence, group), the selection held fixed.
    q_rows [n, Hg, d] (bf16 bits), K, V [L, d] (bf16 bits), sel [n, k] or None (every key u <= t),
    dO [n, Hg, d] (float64). Returns (dQ [n, Hg, d], dK [L, d], dV [L, d]) in float64, dK and dV
    summed over every row and head. Rows are split over threads, each with its own key-gradient
    sums, added in row order at the end."""
    t = _c(t, np.int64)
    q = _c(q_rows, np.uint16)
    K, V = _c(K, np.uint16), _c(V, np.uint16)
    g = _c(dO, np.float64)
    n, Hg, d = q.shape
    dQ = np.zeros((n, Hg, d), np.float64)

    def rows(lo, hi):
        # each worker sums its rows' key gradients into its own arrays
        dK = np.zeros(K.shape, np.float64)
        dV = np.zeros(V.shape, np.float64)
        for r in range(lo, hi):
            s = None if sel is None else _c(sel[r], np.int32)
            ns = 0 if s is None else int((s >= 0).sum())
            for h in range(Hg):
                out = np.zeros(d, np.float64)
                lib().oracle_attend_row_grad(_p(np.ascontiguousarray(q[r, h])), _p(K), _p(V), d, int(t[r]), _p(s), ns,
                                             Bk, _p(np.ascontiguousarray(g[r, h])), _p(out), _p(dK), _p(dV))
                dQ[r, h] = out
        return dK, dV

    nth = max(1, min(nthreads or default_threads(), n))
    bounds = [(i * n // nth, (i + 1) * n // nth) for i in range(nth)]
    if nth == 1:
        parts = [rows(0, n)]
    else:
        import concurrent.futures
        with concurrent.futures.ThreadPoolExecutor(max_workers=nth) as ex:
            parts = list(ex.map(lambda b: rows(*b), bounds))
    dK = np.zeros(K.shape, np.float64)
    dV = np.zeros(V.shape, np.float64)
    for pk, pv in parts:                # in row order, so the result does not depend on threads
        dK += pk
        dV += pv
    return dQ, dK, dV


def e4m3_to_f64(codes) -> np.ndarray:
    """Values of e4m3 codes (uint8), by the format's definition."""
    c = np.asarray(codes, np.uint8)
    return np.array([lib().oracle_e4m3_to_f64(int(v)) for v in c.ravel()], np.float64).reshape(c.shape)


def e4m3_from_f32(x) -> np.ndarray:
    """Nearest e4m3 codes of fp32 values (ties to even mantissa, saturating at +-448)."""
    a = np.asarray(x, np.float32)
    return np.array([lib().oracle_e4m3_from_f32(float(v)) for v in a.ravel()], np.uint8).reshape(a.shape)


def fp8_quantize_blocks(x_bits: np.ndarray, Bk: int = 128):
    """Per-block e4m3 quantisation of bf16 rows [L, d]: (codes [L, d] uint8, scales [ceil(L/Bk)]
    fp32), one scale per block of Bk rows."""
    x = _c(x_bits, np.uint16)
    L, d = x.shape
    codes = np.zeros((L, d), np.uint8)
    nb = (L + Bk - 1) // Bk
    scales = np.zeros(nb, np.float32)
    for j in range(nb):
        blk = np.ascontiguousarray(x[j * Bk:(j + 1) * Bk])
        out = np.zeros(blk.shape, np.uint8)
        scales[j] = lib().oracle_fp8_quantize_block(_p(blk), blk.size, _p(out))
        codes[j * Bk:(j + 1) * Bk] = out
    return codes, scales


def attend_row_fp8(t: int, q_rows: np.ndarray, Kc: np.ndarray, Vc: np.ndarray, ks: np.ndarray,
                   vs: np.ndarray, K: np.ndarray, V: np.ndarray, sel: Optional[np.ndarray] = None,
                   Bk: int = 128):
    """Attention of the query heads q_rows [Hg, d] (bf16 bits) at position t over the FP8 cache
    (codes Kc, Vc [L, d], scales ks, vs per block) with the query's own block from the bf16 rows
    K, V [L, d]. Returns (o [Hg, d], lse [Hg], keys attended)."""
    q = _c(q_rows, np.uint16)
    Kc, Vc = _c(Kc, np.uint8), _c(Vc, np.uint8)
    ks, vs = _c(ks, np.float32), _c(vs, np.float32)
    K, V = _c(K, np.uint16), _c(V, np.uint16)
    Hg, d = q.shape
    s = None if sel is None else _c(sel, np.int32)
    ns = 0 if s is None else int((s >= 0).sum())
    o = np.zeros((Hg, d), np.float64)
    lse = np.zeros(Hg, np.float64)
    nk = 0
    for h in range(Hg):
        oh = np.zeros(d, np.float64)
        lh = np.zeros(1, np.float64)
        nk = lib().oracle_attend_row_fp8(_p(np.ascontiguousarray(q[h])), _p(Kc), _p(Vc), _p(ks), _p(vs),
                                         _p(K), _p(V), d, t, _p(s), ns, Bk, _p(oh), _p(lh))
        o[h], lse[h] = oh, lh[0]
    return o, lse, int(nk)


def select_rows(t: np.ndarray, q_idx_rows: np.ndarray, pooled_g: np.ndarray, Bk: int = 128,
                topk: int = 16, nthreads: Optional[int] = None):
    """Selection for queries of one (sequence, group). Returns (sel [n,topk], kth [n], nsel [n])."""
    t = _c(t, np.int64)
    q = _c(q_idx_rows, np.uint16)
    pg = _c(pooled_g, np.float64)
    n = len(t)
    sel = np.zeros((n, topk), np.int32)
    kth = np.zeros(n, np.float64)
    nsel = np.zeros(n, np.int64)
    lib().oracle_select_rows(n, _p(t), _p(q), _p(pg), q.shape[-1], Bk, topk,
                             nthreads or default_threads(), _p(sel), _p(kth), _p(nsel))
    return sel, kth, nsel


def attend_rows(t: np.ndarray, q_rows: np.ndarray, K: np.ndarray, V: np.ndarray,
                sel: Optional[np.ndarray], Bk: int = 128, topk: int = 16, dense: bool = False,
                nthreads: Optional[int] = None):
    """Attention for queries of one (sequence, group).
    q_rows [n, Hg, d]; K, V [L, d] of the group; sel [n, topk] (ignored when dense).
    Returns (o [n, Hg, d] f64, lse [n, Hg] f64, nkeys [n])."""
    t = _c(t, np.int64)
    q = _c(q_rows, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    n, Hg, d = q.shape
    s = _c(sel if sel is not None else np.full((n, topk), -1), np.int32)
    o = np.zeros((n, Hg, d), np.float64)
    lse = np.zeros((n, Hg), np.float64)
    nk = np.zeros(n, np.int64)
    lib().oracle_attend_rows(n, _p(t), _p(q), Hg, _p(K), _p(V), d, _p(s), topk, Bk,
                             1 if dense else 0, nthreads or default_threads(), _p(o), _p(lse),
                             _p(nk))
    return o, lse, nk


# --------------------------------------------------------------------------- whole passes
def prefill(x: dict, Hq: int, G: int, Bk: int = 128, topk: int = 16, sel: Optional[np.ndarray] = None,
            nthreads: Optional[int] = None, with_attention: bool = True):
    """MSA prefill over whole host tensors (bf16 bits, library layouts):
    q [B,N,Hq,d], k/v [B,G,N,d], q_idx/k_idx [B,N,G,dI].
    If ``sel`` [B,N,G,topk] is given, attention runs on that selection instead of the
    oracle's own. Returns dict(sel, kth, nsel, out [B,N,Hq,d], lse [B,N,Hq], nkeys [B,N,G],
    pooled [B,G,nb,dI])."""
    q, k, v, qi, ki = x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"]
    B, N, _, d = q.shape
    dI = qi.shape[-1]
    Hg = Hq // G
    nb = N // Bk
    t = np.arange(N, dtype=np.int64)
    res = {
        "sel": np.zeros((B, N, G, topk), np.int32),
        "kth": np.zeros((B, N, G), np.float64),
        "nsel": np.zeros((B, N, G), np.int64),
        "pooled": np.zeros((B, G, nb, dI), np.float64),
    }
    if with_attention:
        res["out"] = np.zeros((B, N, Hq, d), np.float64)
        res["lse"] = np.zeros((B, N, Hq), np.float64)
        res["nkeys"] = np.zeros((B, N, G), np.int64)
    for b in range(B):
        pooled, _ = pool(ki[b], Bk)
        res["pooled"][b] = pooled
        for g in range(G):
            s_, kth, ns = select_rows(t, qi[b, :, g, :], pooled[g], Bk, topk, nthreads)
            res["sel"][b, :, g], res["kth"][b, :, g], res["nsel"][b, :, g] = s_, kth, ns
            if with_attention:
                use = s_ if sel is None else sel[b, :, g]
                o, lse, nk = attend_rows(t, q[b, :, g * Hg:(g + 1) * Hg, :], k[b, g], v[b, g],
                                         use, Bk, topk, False, nthreads)
                res["out"][b, :, g * Hg:(g + 1) * Hg] = o
                res["lse"][b, :, g * Hg:(g + 1) * Hg] = lse
                res["nkeys"][b, :, g] = nk
    return res


def prefill_chunk(q: np.ndarray, q_idx: np.ndarray, k_idx: np.ndarray, K: np.ndarray, V: np.ndarray, P: int,
                  Hq: int, G: int, Bk: int = 128, topk: int = 16, sel: Optional[np.ndarray] = None,
                  nthreads: Optional[int] = None):
    """A chunk of a chunked prefill for one sequence: the n queries at positions P .. P + n - 1
    against everything up to P + n - 1 (youmind article "MiniMax M3 sparse attention agents",
    bullet "Predictable cost at every length": the same 16-block budget at every length).
    Steps 1-4 exactly as in a whole prefill, at those positions: pooled keys of every full block
    below P + n, selection among the fully-past blocks, attention over the selected keys u <= t.
    q [n, Hq, d], q_idx [n, G, dI] (the chunk's rows); k_idx [>= P + n, G, dI], K, V [G, >= P + n, d]
    (the sequence so far, the chunk included). If ``sel`` [n, G, topk] is given, attention runs on
    it. Returns dict(sel [n,G,topk], kth [n,G], pooled [G,nb,dI], out [n,Hq,d], lse [n,Hq])."""
    n = q.shape[0]
    Hg = Hq // G
    t = np.arange(P, P + n, dtype=np.int64)
    pooled, _ = pool(k_idx[:P + n], Bk)
    res = {"sel": np.zeros((n, G, topk), np.int32), "kth": np.zeros((n, G), np.float64), "pooled": pooled,
           "out": np.zeros((n, Hq, q.shape[-1]), np.float64), "lse": np.zeros((n, Hq), np.float64)}
    for g in range(G):
        s_, kth, _ = select_rows(t, q_idx[:, g, :], pooled[g], Bk, topk, nthreads)
        res["sel"][:, g], res["kth"][:, g] = s_, kth
        use = s_ if sel is None else sel[:, g]
        o, lse, _ = attend_rows(t, q[:, g * Hg:(g + 1) * Hg, :], K[g], V[g], use, Bk, topk, False, nthreads)
        res["out"][:, g * Hg:(g + 1) * Hg] = o
        res["lse"][:, g * Hg:(g + 1) * Hg] = lse
    return res


def dense_gqa(x: dict, Hq: int, G: int, nthreads: Optional[int] = None):
    """Dense causal GQA attention (every key u <= t) with the same layouts; the comparator
    the pages measure MSA against. Returns (out [B,N,Hq,d], lse [B,N,Hq])."""
    q, k, v = x["q"], x["k"], x["v"]
    B, N, _, d = q.shape
    Hg = Hq // G
    t = np.arange(N, dtype=np.int64)
    out = np.zeros((B, N, Hq, d), np.float64)
    lse = np.zeros((B, N, Hq), np.float64)
    for b in range(B):
        for g in range(G):
            o, l, _ = attend_rows(t, q[b, :, g * Hg:(g + 1) * Hg, :], k[b, g], v[b, g], None,
                                  dense=True, nthreads=nthreads)
            out[b, :, g * Hg:(g + 1) * Hg] = o
            lse[b, :, g * Hg:(g + 1) * Hg] = l
    return out, lse
