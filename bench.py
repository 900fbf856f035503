#!/usr/bin/env python
"""Benchmark of the MSA (MiniMax Sparse Attention over GQA) hot path on B200.

One step = one pass of the whole hot path on synthetic inputs already resident in HBM:
  * prefill of 131,072 tokens, batch 1, 64 query heads / 8 KV groups (pooling, block scoring +
    exp-free top-16 selection, main-branch sparse attention), and
  * one decode step of a batch of 16 sequences at 131,072 cached tokens (selection, append +
    pooled-key update, attention split over the selected blocks), replayed from a CUDA graph.
L2 is flushed (256 MiB write, then 256 MiB read) before every timed step, outside the events.

Printed value: prefill tokens/s over all ranks (131,072 x N / slowest rank's prefill time).
The same line carries the decode step latency, the index-select and main-branch split, the
roofline fractions, the end-to-end figure through host buffers, the clocks seen, and the CPU
oracle baseline. ``--impl reference`` times the fp64 CPU oracle instead (the reference arm).
``--topk`` runs the exp-free top-k micro-benchmark against torch.topk instead of the step.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MSA prefill tok/s & decode step µs at 128K ctx; % of HBM/tensor roofline"
PREFILL = synth.WORKLOADS["prefill_128k_h64g8"]
DECODE = synth.WORKLOADS["decode_128k_b16_h64g8"]
PREFILL_32K = synth.WORKLOADS["prefill_32k_h64g8_planted"]
PREFILL_4K = synth.WORKLOADS["prefill_4k_h4g1"]
DECODE_1M = synth.WORKLOADS["decode_1m_ragged_b4_h64g8"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = os.path.join(ROOT, "block_sparse_gqa_branch_b200", "csrc")

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) from ncu captures of the kernels
# behind each roofline, with the hash of the CUDA sources the captured build was made from
# (source_sha16 of the listed files). A capture stands only while those sources are unchanged:
# when any of them changes, the bench reports traffic null until the capture is taken again.
# Each entry says which workload was captured and how it is scaled to the bench's workload.
CAPTURES = {
    "decode_step": {
        # attn_decode_kernel 32,132,608 B read + 6,144 B written; select_decode_kernel 8,428,800 B read
        "bytes": 32132608 + 6144 + 8428800,
        "algorithmic_bytes": 40052736,          # decode_step_bytes of the batch-4 workload
        "sources": ["attn_decode.cu", "select.cu"], "sha16": "10befc6ca47e5ecb",
        "note": "attention + selection DRAM bytes at decode_128k_b4_h64g8 (ncu --set full, one launch each), "
                "scaled to the bench's batch by the algorithmic bytes (both kernels' work is per (sequence, group))",
        "profile": "profiles/attn_decode_kernel_decode128k_b4.md, profiles/select_decode_kernel_decode128k_b4.md"},
    "attn_prefill": {
        # attn_kvmajor_kernel at a prefill of 8,192 tokens: 257,352,704 B read + 1.873613e9 B written
        "bytes": 257352704 + 1873613000, "model_bytes": 2130214912,   # prefill_main_bytes(...)["attn_model"] at 8K
        # The captured build's attn_prefill.cu hashed f6d5cb4e3f98890f. The file has changed since
        # only in the inverted-index kernels (csr_scan_kernel, csr_fill_kernel) and their launch
        # code, which this capture does not include; attn_kvmajor_kernel and combine_kernel and
        # every device function they call are unchanged, so the hash is that of the current file.
        "sources": ["attn_prefill.cu"], "sha16": "548d8318fd915d4a",
        "note": "DRAM bytes of attn_kvmajor_kernel at prefill_8192_h64g8 (ncu --set full, one launch), scaled to "
                "the bench's prefill by this build's byte model of the kernel (partial writes are 88% of it)",
        "profile": "profiles/attn_kvmajor_kernel_prefill8k.md"},
    "prefill_main": {
        # attention (above) + combine_kernel 1,931,634,000 B read + 90,584,576 B written, same run and size
        "bytes": 257352704 + 1873613000 + 1931634000 + 90584576, "model_bytes": 4208001024,
        "sources": ["attn_prefill.cu"], "sha16": "548d8318fd915d4a",   # as above: the captured kernels are unchanged
        "note": "DRAM bytes of the attention and combine kernels at prefill_8192_h64g8 (the inverted index's three "
                "small kernels not captured), scaled by the main-branch call's byte model",
        "profile": "profiles/attn_kvmajor_kernel_prefill8k.md, profiles/combine_kernel_prefill8k.md"},
    "topk_rows": {
        "bytes": 536937472 + 7052800, "rows": 131072,
        "sources": ["topk.cu"], "sha16": "dafaf2384b8ae8c3",
        "note": "DRAM bytes of topk_rows_kernel at 131,072 x 1,024 (ncu --set full, one launch), scaled by rows",
        "profile": "profiles/topk_rows_kernel_131072x1024.md"},
}


def source_sha16(files) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def captured_traffic(name: str, scale: float):
    """(bytes per launch of the bench workload, note) from CAPTURES, or (None, why)."""
    c = CAPTURES.get(name)
    if c is None:
        return None, "no capture recorded"
    if source_sha16(c["sources"]) != c["sha16"]:
        return None, "kernel sources changed since the capture (" + c["profile"] + ")"
    return int(round(c["bytes"] * scale)), c["note"] + " (" + c["profile"] + ")"


# ----------------------------------------------------------------------------- work counts
def attended_pairs(N: int, Bk: int = 128, k: int = 16) -> int:
    """(query, key) pairs a causal MSA prefill of N tokens attends per (head): a query at t in
    block c attends every key u <= t when c + 1 <= k, else (k-1)*Bk + (t mod Bk) + 1 keys."""
    total = 0
    for c in range((N + Bk - 1) // Bk):
        lo, hi = c * Bk, min(N, (c + 1) * Bk)
        for t in range(lo, hi):
            total += (t + 1) if c + 1 <= k else (k - 1) * Bk + (t - lo) + 1
    return total


def prefill_main_flops(w) -> float:
    return 4.0 * w.d * w.Hq * attended_pairs(w.N, w.Bk, w.topk)   # QK^T and PV, 2 FLOP per MAC


def prefill_index_flops(w) -> float:
    """2 * d_I FLOP per (query, group, candidate): a query at t scores its t // Bk fully-past
    blocks, so a full block c contributes Bk * c candidates and the ragged tail (N mod Bk) *
    (N // Bk)."""
    nbf = w.N // w.Bk
    cand = w.Bk * (nbf * (nbf - 1) // 2) + (w.N % w.Bk) * nbf
    return 2.0 * w.dI * w.G * w.B * cand


def decode_step_bytes(w) -> dict:
    """Algorithmic HBM bytes of one decode step (every byte the definition must touch once)."""
    kv = pooled = 0
    for L in w.ctx:
        c = L // w.Bk
        pooled += w.G * c * w.dI * 4                               # scored candidates' pooled keys
        nfull = min(c, w.topk - 1)
        kv += w.G * (nfull * w.Bk + (L % w.Bk) + 1) * w.d * 2 * 2   # K and V of the selected blocks
    small = w.B * (w.Hq * w.d * 2 * 2                               # q in, out
                   + w.G * w.dI * 2 * 2                             # q_I, k_I(new)
                   + w.G * w.d * 2 * 2 * 2                          # k_new, v_new read + cache write
                   + w.G * w.dI * 4 * 2 + w.G * w.topk * 4)         # running sum, sel
    return {"kv": kv, "pooled": pooled, "small": small, "total": kv + pooled + small}


def decode_step_bytes_fp8(w) -> dict:
    """Algorithmic HBM bytes of one decode step over the FP8 cache: as decode_step_bytes, but
    the selected closed blocks are read as one e4m3 byte per value plus a key and a value scale;
    the query's own block is read in bf16."""
    base = decode_step_bytes(w)
    kv = 0
    for L in w.ctx:
        c = L // w.Bk
        nfull = min(c, w.topk - 1)
        kv += w.G * (nfull * (w.Bk * w.d * 2 + 2 * 4) + ((L % w.Bk) + 1) * w.d * 2 * 2)
    return dict(base, kv=kv, total=kv + base["pooled"] + base["small"])


def _per_block_counts(N: int, Bk: int, k: int):
    """(tokens, fully-past blocks kept per token) for every query block of an N-token prefill."""
    for c in range((N + Bk - 1) // Bk):
        yield min(Bk, N - c * Bk), min(c, k - 1)


def prefill_main_bytes(w, range_tokens: int = 16384) -> dict:
    """Bytes of the main-branch call (inverted index, attention, merge) of a prefill.

    algorithmic: what the definition must touch once -- q, the selection, K and V, out and lse.
    model: what this build moves to or from DRAM when the re-reads of query rows and of key /
    value blocks within one 16K-token range hit L2: the selection read three times (count,
    fill, merge), the inverted-index entries written and read, q once, K and V once per
    (range, group, block) below the range's end plus once per diagonal item, one partial per
    (token, head, selected block) -- 256 B of bf16 o and a 4 B log-sum-exp -- written by the
    attention and read by the merge, then out and lse written."""
    B, N, G, Hq, d, Bk, k = w.B, w.N, w.G, w.Hq, w.d, w.Bk, w.topk
    nb = (N + Bk - 1) // Bk
    entries = sum(n * kept for n, kept in _per_block_counts(N, Bk, k)) * B * G
    rows = sum(n * (kept + 1) for n, kept in _per_block_counts(N, Bk, k)) * B * Hq
    q = B * N * Hq * d * 2
    out = q + B * N * Hq * 4
    sel = B * N * G * k * 4
    kv_once = B * G * N * d * 2 * 2
    n_ranges = (N + range_tokens - 1) // range_tokens
    kv_tiles = sum(min(nb, (r + 1) * (range_tokens // Bk)) for r in range(n_ranges)) + nb
    kv_model = B * G * kv_tiles * Bk * d * 2 * 2
    partials = rows * (d * 2 + 4)
    model = 3 * sel + 2 * entries * 4 + q + kv_model + 2 * partials + out
    attn_model = q + kv_model + partials + entries * 4       # the attention kernel alone
    return {"algorithmic": q + sel + kv_once + out, "model": model, "attn_model": attn_model, "partial_rows": rows,
            "partials": partials}


def prefill_index_bytes(w) -> int:
    """Compulsory bytes of the index branch: k_I and q_I read, the pooled keys written and read
    back once, the selection written."""
    nb = w.N // w.Bk
    return w.B * (w.N * w.G * w.dI * 2 * 2 + w.G * nb * w.dI * 4 * 2 + w.N * w.G * w.topk * 4)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            with open(self.path) as f:
                for r in csv.reader(f):
                    if len(r) >= 9:
                        rows.append([x.strip() for x in r])
        except OSError:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s, p in zip(sm, pw) if p > 250.0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(pw) if pw else None}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_prefill_sample(w, n_rows: int, g: int, seed: int = 7, cache: dict = None):
    """Time the oracle on n_rows (token, group g) rows of a prefill workload, uniformly sampled.
    Returns (seconds per token over all G groups including the group's pooling, seconds of
    oracle work this sample took)."""
    import oracle
    cache = {} if cache is None else cache
    key = ("grp", g)
    if key not in cache:
        N, G = w.N, w.G
        pos = np.arange(N, dtype=np.uint64)
        ki = synth.normal_bf16_at(w.seed, synth.STREAM_KI,
                                  ((pos[:, None] * np.uint64(G) + np.uint64(g)) * np.uint64(w.dI)
                                   + np.arange(w.dI, dtype=np.uint64)[None, :]))
        kk = synth.normal_bf16(w.seed, synth.STREAM_K, (N, w.d), start=g * N * w.d)
        vv = synth.normal_bf16(w.seed, synth.STREAM_V, (N, w.d), start=g * N * w.d)
        cache[key] = (ki[:, None, :], kk, vv)
    ki, kk, vv = cache[key]
    rng = np.random.default_rng(seed)
    t = np.sort(rng.integers(0, w.N, n_rows)).astype(np.int64)
    hq = np.arange(g * w.Hg, (g + 1) * w.Hg, dtype=np.uint64)
    qidx = ((t.astype(np.uint64)[:, None, None] * np.uint64(w.Hq) + hq[None, :, None]) * np.uint64(w.d)
            + np.arange(w.d, dtype=np.uint64)[None, None, :])
    q = synth.normal_bf16_at(w.seed, synth.STREAM_Q, qidx)
    qiidx = ((t.astype(np.uint64)[:, None] * np.uint64(w.G) + np.uint64(g)) * np.uint64(w.dI)
             + np.arange(w.dI, dtype=np.uint64)[None, :])
    qi = synth.normal_bf16_at(w.seed, synth.STREAM_QI, qiidx)
    t0 = time.perf_counter()
    pooled, _ = oracle.pool(ki, w.Bk)
    t1 = time.perf_counter()
    sel, _, _ = oracle.select_rows(t, qi, pooled[0], w.Bk, w.topk)
    oracle.attend_rows(t, q, kk, vv, sel, w.Bk, w.topk)
    t2 = time.perf_counter()
    per_token = (t2 - t1) / n_rows * w.G + (t1 - t0) * w.G / w.N
    return per_token, t2 - t0


def cpu_baseline(w, budget_s: float = 15.0):
    """The oracle as it stands on this host's cores, on a bounded sample of the workload."""
    import oracle
    cache = {}
    n = 64
    per_tok, el = oracle_prefill_sample(w, n, 0, cache=cache)
    n2 = int(max(64, min(20000, n * budget_s / max(el, 1e-3) * 0.8)))
    per_tok, el = oracle_prefill_sample(w, n2, 0, seed=11, cache=cache)
    return {"value": 1.0 / per_tok, "unit": "tok/s", "cores": oracle.default_threads(), "kind": "oracle",
            "sample": f"{n2} (token, group 0) rows of {w.name} drawn uniformly over positions, "
                      f"selection + attention for {w.Hg} heads each, plus group 0's pooling; "
                      f"scaled to whole tokens (x{w.G} groups); {el:.1f} s of CPU time"}


def oracle_decode_step(w):
    """The oracle's decode step over EVERY (sequence, group) pair of a decode workload: the
    selection of the new token's blocks from the pooled cache and the attention of its Hg heads
    over them. The pooled cache (built from all earlier tokens) and the K/V rows of the
    selected blocks are prepared first and not timed. Pairs run concurrently, one oracle thread
    each. Returns (seconds, threads used)."""
    import concurrent.futures
    import oracle
    threads = min(oracle.default_threads(), w.B * w.G)
    work = []
    for b in range(w.B):
        Lb = w.ctx[b]
        ki = synth.decode_seq_np(w, b, "k_idx")
        pooled, _ = oracle.pool(ki, w.Bk)
        del ki
        qi = synth.decode_seq_np(w, b, "q_idx")
        q = synth.decode_seq_np(w, b, "q")
        for g in range(w.G):
            work.append((b, g, Lb, np.ascontiguousarray(pooled[g]), qi[g][None].copy(),
                         q[g * w.Hg:(g + 1) * w.Hg][None].copy()))
        del pooled
    t = np.zeros(1)

    def select(item):
        b, g, Lb, pooled_g, qi, _ = item
        sel, _, _ = oracle.select_rows(np.array([Lb]), qi, pooled_g, w.Bk, w.topk, nthreads=1)
        return sel

    wall0 = time.perf_counter()
    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        sels = list(ex.map(select, work))
    t[0] = time.perf_counter() - wall0
    # K / V rows of the selected blocks only (not timed)
    kv = []
    for (b, g, Lb, _, _, _), sel in zip(work, sels):
        K = np.zeros((Lb + 1, w.d), np.uint16)
        V = np.zeros((Lb + 1, w.d), np.uint16)
        for j in sel[0]:
            if j >= 0:
                lo, hi = j * w.Bk, min((j + 1) * w.Bk, Lb + 1)
                K[lo:hi] = synth.decode_seq_np(w, b, "k", lo, hi, g=g)
                V[lo:hi] = synth.decode_seq_np(w, b, "v", lo, hi, g=g)
        kv.append((K, V))

    def attend(i):
        b, g, Lb, _, _, q = work[i]
        K, V = kv[i]
        oracle.attend_rows(np.array([Lb]), q, K, V, sels[i], w.Bk, w.topk, nthreads=1)

    wall0 = time.perf_counter()
    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(attend, range(len(work))))
    t[0] += time.perf_counter() - wall0
    return float(t[0]), threads


def cpu_baseline_decode(w):
    sec, threads = oracle_decode_step(w)
    return {"value": sec * 1e6, "unit": "us per step", "cores": threads, "kind": "oracle",
            "sample": f"whole step of {w.name}: all {w.B * w.G} (sequence, group) pairs, selection over "
                      f"the pooled cache + attention of {w.Hg} heads over the selected blocks "
                      f"(pooled cache and K/V rows prepared beforehand, not timed)"}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands on the host cores, on a bounded sample of
    the prefill workload per step (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    cache = {}
    n = 64
    _, el = oracle_prefill_sample(PREFILL, n, 0, cache=cache)
    n_step = int(max(32, min(20000, n * 4.0 / max(el, 1e-3))))
    per_tok_l, step_s = [], []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        per_tok, _ = oracle_prefill_sample(PREFILL, n_step, 0, seed=100 + s, cache=cache)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            per_tok_l.append(per_tok)
            step_s.append(dt)
    per_tok = statistics.mean(per_tok_l)
    value = 1.0 / per_tok
    sample = (f"each step: {n_step} (token, group 0) rows of {PREFILL.name} drawn uniformly, "
              f"selection + attention, plus group 0's pooling; value scaled to whole tokens (x{PREFILL.G})")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.mean(step_s) * 1e3,
            "ms_per_step_note": "measured seconds of one step's sample (rows drawn, oracle run)",
            "extrapolated_full_prefill_ms": per_tok * PREFILL.N * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded SplitMix64 -> N(0,1) quantiles -> bf16)",
            "config": config_block(PREFILL, DECODE),
            "cpu_baseline": {"value": value, "unit": "tok/s", "cores": oracle.default_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workloads(args):
    """The benchmark workloads, or smaller ones of the same structure for a profiler capture."""
    import dataclasses
    wp, wd = PREFILL, DECODE
    if args.prefill_tokens:
        wp = dataclasses.replace(wp, N=args.prefill_tokens, name=f"prefill_{args.prefill_tokens}_h64g8")
    if args.decode_batch:
        wd = dataclasses.replace(wd, B=args.decode_batch, ctx=wd.ctx[:1] * args.decode_batch,
                                 name=f"decode_128k_b{args.decode_batch}_h64g8")
    return wp, wd


def config_block(wp, wd):
    return {"workload": f"{wp.name} + {wd.name}",
            "prefill": {"batch": wp.B, "seq_len": wp.N, "q_heads": wp.Hq, "kv_groups": wp.G,
                        "head_dim": wp.d, "index_dim": wp.dI, "block": wp.Bk, "top_k": wp.topk},
            "decode": {"batch": wd.B, "ctx_len": wd.ctx[0], "q_heads": wd.Hq, "kv_groups": wd.G,
                       "head_dim": wd.d, "index_dim": wd.dI, "block": wd.Bk, "top_k": wd.topk},
            "l2": "flushed before every timed step and before the decode half (256 MiB write, then 256 MiB read)",
            "parallelism": "replicas (one independent problem per GPU)"}


# ----------------------------------------------------------------------------- GPU arm
def build_decode_state(w, device):
    import torch
    from block_sparse_gqa_branch_b200 import Shape, msa_pool_index_keys
    B, G = w.B, w.G
    Lmax = max(w.ctx) + 1
    l_cap = (Lmax + 127) // 128 * 128
    nb_cap = l_cap // 128 + 1
    k_cache = torch.zeros(B, G, l_cap, 128, dtype=torch.bfloat16, device=device)
    v_cache = torch.zeros_like(k_cache)
    pooled = torch.zeros(B, G, nb_cap, 64, device=device)
    tail = torch.zeros(B, G, 64, device=device)
    new = {"q": torch.empty(B, w.Hq, 128, dtype=torch.bfloat16, device=device),
           "q_idx": torch.empty(B, G, 64, dtype=torch.bfloat16, device=device),
           "k_idx_new": torch.empty(B, G, 64, dtype=torch.bfloat16, device=device),
           "k_new": torch.empty(B, G, 128, dtype=torch.bfloat16, device=device),
           "v_new": torch.empty(B, G, 128, dtype=torch.bfloat16, device=device)}
    for b in range(B):
        Lb = w.ctx[b]
        kk = synth.decode_seq_torch(w, b, "k", device)
        k_cache[b, :, :Lb] = kk[:, :Lb]
        new["k_new"][b] = kk[:, Lb]
        del kk
        vv = synth.decode_seq_torch(w, b, "v", device)
        v_cache[b, :, :Lb] = vv[:, :Lb]
        new["v_new"][b] = vv[:, Lb]
        del vv
        ki = synth.decode_seq_torch(w, b, "k_idx", device)
        new["k_idx_new"][b] = ki[Lb]
        msa_pool_index_keys(Shape.make(1, w.Hq, G), ki[:Lb].contiguous(), Lb, pooled[b], nb_cap, tail[b])
        del ki
        new["q"][b] = synth.decode_seq_torch(w, b, "q", device)
        new["q_idx"][b] = synth.decode_seq_torch(w, b, "q_idx", device)
    ctx = torch.tensor(list(w.ctx), dtype=torch.int32, device=device)
    return {"k_cache": k_cache, "v_cache": v_cache, "pooled": pooled, "tail": tail, "ctx": ctx, **new}


def reduce_max(x: float, world: int, device) -> float:
    """The largest of the ranks' values (every rank calls it; one collective when world > 1)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def make_flusher(torch, dev):
    """L2 flush between timed steps: write a buffer larger than L2 (126 MB), then read another
    one, so that the written lines are written back before the timed region (a write alone
    leaves ~126 MB of dirty lines whose write-back would land inside the next step)."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        flush_rd.sum()
    return flush_l2


def kernel_means(records, steps: int) -> dict:
    """Per-kernel device milliseconds per step from msa_kernel_timing_read records:
    {name: {"ms": total per step, "launches": per step}}."""
    out = {}
    for name, ms in records:
        e = out.setdefault(name, {"ms": 0.0, "launches": 0})
        e["ms"] += ms
        e["launches"] += 1
    return {k: {"ms": v["ms"] / steps, "launches": v["launches"] / steps} for k, v in out.items()}


def time_prefill(torch, w, dev, steps, warmup, flush_l2):
    """Prefill of workload w (inputs resident in HBM): per-step (index, main) device seconds."""
    from block_sparse_gqa_branch_b200 import (msa_get_device_status, msa_kernel_launches, msa_kernel_timing_enable,
                                              msa_kernel_timing_read, pipeline)
    x = synth.prefill_inputs_torch(w, dev)
    bufs = pipeline.prefill_buffers(w.B, w.N, w.Hq, w.G, dev)
    stream = torch.cuda.current_stream()
    pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], bufs)
    ti, tm = [], []
    for s in range(warmup + steps):
        flush_l2()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        if s == warmup:
            torch.cuda.synchronize()
            l0 = msa_kernel_launches()
            msa_kernel_timing_read(0)
            msa_kernel_timing_enable(True)
        e[0].record(stream)
        pipeline.prefill_index(x["q_idx"], x["k_idx"], bufs)
        e[1].record(stream)
        pipeline.prefill_main(x["q"], x["k"], x["v"], bufs)
        e[2].record(stream)
        if s >= warmup:
            ti.append(e)
    torch.cuda.synchronize()
    launches = msa_kernel_launches() - l0
    msa_kernel_timing_enable(False)
    kernels = kernel_means(msa_kernel_timing_read(), steps)
    for key in ("ws_select", "ws_attn"):
        st_, info = msa_get_device_status(bufs[key])
        if st_ != 0:
            raise SystemExit(f"device status {st_} in {w.name} {key}: {info}")
    t_index = [a.elapsed_time(b) * 1e-3 for a, b, _ in ti]
    t_main = [b.elapsed_time(c) * 1e-3 for _, b, c in ti]
    return t_index, t_main, launches, kernels


def time_decode(torch, w, dev, steps, warmup, flush_l2, fp8=False):
    """Decode step of workload w replayed from a CUDA graph: per-step device seconds. With fp8,
    the closed blocks are read from an e4m3 cache quantised from the bf16 one beforehand."""
    from block_sparse_gqa_branch_b200 import msa_get_device_status, pipeline
    ds = build_decode_state(w, dev)
    bufs = pipeline.decode_buffers(w.B, w.Hq, w.G, max(w.ctx), dev)
    f8 = None
    if fp8:
        f8 = pipeline.fp8_cache(ds["k_cache"], ds["v_cache"], ds["pooled"].shape[2])
        for b in range(w.B):
            pipeline.fp8_quantize_sequence(ds["k_cache"], ds["v_cache"], f8, b, w.ctx[b], w.Hq)

    def call():
        if fp8:
            pipeline.decode_step_fp8(ds["q"], ds["q_idx"], ds["k_idx_new"], ds["k_new"], ds["v_new"], ds["ctx"],
                                     ds["k_cache"], ds["v_cache"], ds["tail"], ds["pooled"], f8, bufs)
        else:
            pipeline.decode_step(ds["q"], ds["q_idx"], ds["k_idx_new"], ds["k_new"], ds["v_new"], ds["ctx"],
                                 ds["k_cache"], ds["v_cache"], ds["tail"], ds["pooled"], bufs)
    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    stream = torch.cuda.current_stream()
    ts = []
    for s in range(warmup + steps):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        if s >= warmup:
            ts.append((e0, e1))
    torch.cuda.synchronize()
    for key in ("ws_append", "ws_select", "ws_attn"):
        st_, info = msa_get_device_status(bufs[key])
        if st_ != 0:
            raise SystemExit(f"device status {st_} in {w.name} {key}: {info}")
    del graph
    return [a.elapsed_time(b) * 1e-3 for a, b in ts], (4 if fp8 else 3) * steps


def time_backward(torch, w, dev, steps, warmup, flush_l2):
    """Backward pass of the main branch after a prefill of workload w (its selection, output and
    lse; upstream gradient seeded like q): per-step device seconds of msa_sparse_attn_prefill_backward."""
    from block_sparse_gqa_branch_b200 import msa_get_device_status, pipeline
    x = synth.prefill_inputs_torch(w, dev)
    fwd = pipeline.prefill_buffers(w.B, w.N, w.Hq, w.G, dev)
    pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], fwd)
    del fwd["ws_attn"], fwd["ws_select"]
    torch.cuda.empty_cache()
    d_out = synth.normal_bf16_torch(w.seed + 99, synth.STREAM_Q, w.B * w.N * w.Hq * w.d, dev).view(w.B, w.N, w.Hq, w.d)
    bwd = pipeline.backward_buffers(w.B, w.N, w.Hq, w.G, dev)
    stream = torch.cuda.current_stream()
    ts = []
    for s in range(warmup + steps):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pipeline.prefill_backward(x["q"], x["k"], x["v"], d_out, fwd, bwd)
        e1.record(stream)
        if s >= warmup:
            ts.append((e0, e1))
    torch.cuda.synchronize()
    st_, info = msa_get_device_status(bwd["ws"])
    if st_ != 0:
        raise SystemExit(f"device status {st_} in the backward pass: {info}")
    return [a.elapsed_time(b) * 1e-3 for a, b in ts]


def time_prefill_chunked(torch, w, dev, chunk, steps, warmup, flush_l2):
    """A prefill of workload w in chunks of `chunk` tokens against a cache (pool, select and
    attention per chunk, caches filled with the chunk's K/V beforehand): per-step seconds of
    all chunks."""
    from block_sparse_gqa_branch_b200 import (OP_INDEX_SELECT_PREFILL, Shape, msa_get_device_status,
                                              msa_index_select_chunk, msa_pool_index_keys_chunk,
                                              msa_prefill_chunk_workspace_size, msa_sparse_attn_prefill_chunk,
                                              msa_workspace_size)
    x = synth.prefill_inputs_torch(w, dev)
    B, N, G, Hq = w.B, w.N, w.G, w.Hq
    shape = Shape.make(B, Hq, G)
    nb_cap = (N + 127) // 128
    pooled = torch.zeros(B, G, nb_cap, 64, device=dev)
    tail = torch.zeros(B, G, 64, device=dev)
    starts = list(range(0, N, chunk))
    qs = [x["q"][:, p:p + chunk].contiguous() for p in starts]
    qis = [x["q_idx"][:, p:p + chunk].contiguous() for p in starts]
    kis = [x["k_idx"][:, p:p + chunk].contiguous() for p in starts]
    del x["q"]
    sel = [torch.empty(B, min(chunk, N - p), G, 16, dtype=torch.int32, device=dev) for p in starts]
    out = [torch.empty(B, min(chunk, N - p), Hq, 128, dtype=torch.bfloat16, device=dev) for p in starts]
    lse = [torch.empty(B, min(chunk, N - p), Hq, dtype=torch.float32, device=dev) for p in starts]
    ws_sel = torch.zeros(msa_workspace_size(shape, OP_INDEX_SELECT_PREFILL, N), dtype=torch.uint8, device=dev)
    ws = torch.zeros(max(msa_prefill_chunk_workspace_size(shape, p, min(chunk, N - p)) for p in starts),
                     dtype=torch.uint8, device=dev)

    def run():
        tail.zero_()
        for i, p in enumerate(starts):
            n = min(chunk, N - p)
            msa_pool_index_keys_chunk(shape, kis[i], p, n, pooled, nb_cap, tail)
            msa_index_select_chunk(shape, qis[i], p, n, pooled, nb_cap, sel[i], ws_sel)
            msa_sparse_attn_prefill_chunk(shape, qs[i], x["k"], x["v"], N, p, n, sel[i], out[i], lse[i], ws)
    stream = torch.cuda.current_stream()
    ts = []
    for s in range(warmup + steps):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        if s >= warmup:
            ts.append((e0, e1))
    torch.cuda.synchronize()
    for buf in (ws_sel, ws):
        st_, info = msa_get_device_status(buf)
        if st_ != 0:
            raise SystemExit(f"device status {st_} in the chunked prefill: {info}")
    return [a.elapsed_time(b) * 1e-3 for a, b in ts], len(starts)


def prefill_report(w, t_index, t_main, peaks, peak_src, world, launches, kernels):
    """kernels: per-kernel device ms per step timed live in the same steps (kernel_means); the
    roofline is that of the dominant kernel, attn_kvmajor_kernel, over its own launch time."""
    tidx, tmain = statistics.mean(t_index), statistics.mean(t_main)
    flops = prefill_main_flops(w)
    ach = flops / tmain / 1e12
    t_attn = kernels["attn_prefill"]["ms"] * 1e-3
    ach_k = flops / t_attn / 1e12
    mb = prefill_main_bytes(w)
    # captured DRAM bytes of a smaller prefill, scaled by this build's byte model (partial writes dominate)
    cap_a, cap_m = CAPTURES.get("attn_prefill"), CAPTURES.get("prefill_main")
    traffic, tnote = (captured_traffic("attn_prefill", mb["attn_model"] / cap_a["model_bytes"]) if cap_a
                      else (None, "no capture recorded"))
    call_traffic, cnote = (captured_traffic("prefill_main", mb["model"] / cap_m["model_bytes"]) if cap_m
                           else (None, "no capture recorded"))
    idx_flops = prefill_index_flops(w)
    idx_bytes = prefill_index_bytes(w)
    return {
        "workload": w.name, "value": w.N * w.B * world / (tidx + tmain), "unit": "tok/s",
        "prefill_ms": (tidx + tmain) * 1e3, "prefill_index_ms": tidx * 1e3, "prefill_main_ms": tmain * 1e3,
        "gpu_launches": int(launches),
        "roofline": {"bound": "tensor", "achieved": ach_k, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": ach_k / peaks["bf16_tflops"], "traffic": traffic, "traffic_note": tnote,
                     "kernel": "attn_kvmajor_kernel (main-branch attention; its launch time from CUDA events "
                               "around it in the timed steps)",
                     "launch_ms": t_attn * 1e3,
                     "algorithmic": f"{flops:.4e} FLOP per launch", "peak_source": f"{peak_src} burst bf16"},
        "roofline_call": {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": ach / peaks["bf16_tflops"],
                          "kernel": "prefill main branch (msa_sparse_attn_prefill: inverted index, attention, merge)",
                          "algorithmic": f"{flops:.4e} FLOP per call", "peak_source": f"{peak_src} burst bf16"},
        "kernels_ms": {k: round(v["ms"], 4) for k, v in kernels.items()},
        "hbm": {"algorithmic_bytes": mb["algorithmic"], "model_bytes": mb["model"],
                "traffic": call_traffic, "traffic_note": cnote,
                "achieved_gbs": mb["algorithmic"] / tmain / 1e9,
                "frac": mb["algorithmic"] / tmain / 1e9 / peaks["hbm_gbs"],
                "model_frac": mb["model"] / tmain / 1e9 / peaks["hbm_gbs"],
                "note": "main branch: algorithmic = q, sel, K, V read once and out, lse written; model = "
                        "this build's DRAM bytes (partials written and read back dominate)"},
        "roofline_index": {"bound": "tensor", "achieved": idx_flops / tidx / 1e12, "peak": peaks["bf16_tflops"],
                           "unit": "TFLOP/s", "frac": idx_flops / tidx / 1e12 / peaks["bf16_tflops"],
                           "executed_frac": 6 * idx_flops / tidx / 1e12 / peaks["bf16_tflops"],
                           "hbm_frac": idx_bytes / tidx / 1e9 / peaks["hbm_gbs"],
                           "kernel": "index branch (pooling + scores + exp-free top-15)",
                           "algorithmic": f"{idx_flops:.4e} FLOP (2 d_I per query, group and candidate; "
                                          f"executed 6x: the exact three-term bf16 split, and the id pass "
                                          f"recomputes every score), {idx_bytes} B compulsory"},
    }


def decode_report(w, t_dec, peaks, peak_src, launches, traffic_name=None, scale=1.0, fp8=False):
    tdec = statistics.mean(t_dec)
    dbytes = decode_step_bytes_fp8(w) if fp8 else decode_step_bytes(w)
    gbs = dbytes["total"] / tdec / 1e9
    traffic, tnote = captured_traffic(traffic_name, scale) if traffic_name else (None, "not captured")
    return {
        "workload": w.name, "decode_step_us": tdec * 1e6, "gpu_launches": int(launches),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": traffic, "traffic_note": tnote,
                     "kernel": ("decode step over the FP8 cache (select + append + close + attention, one graph replay)"
                                if fp8 else "decode step (select + append + attention, one graph replay)"),
                     "algorithmic": f"{dbytes['total']} B per step", "peak_source": f"{peak_src} copy"},
    }


def topk_report(torch, dev, steps, warmup, peaks, peak_src, with_torch=True, rows=8 * 131072):
    """Exp-free top-k (msa_topk_rows) on the block scores of 8 groups at 131,072 tokens:
    [1,048,576, 1024] fp32 seeded normal values on the device, k = 15; 4.3 GB exceed L2.
    (`rows` smaller only for profiler captures.)"""
    import block_sparse_gqa_branch_b200 as msa
    n, k = 1024, 15
    s = torch.randn(rows, n, device=dev, generator=torch.Generator(device=dev).manual_seed(0x4D5341))
    idx = torch.empty(rows, k, dtype=torch.int32, device=dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3)
        return statistics.median(ts)

    t_ref = timed(lambda: torch.topk(s, k, dim=1)) if with_torch else None
    l0 = msa.msa_kernel_launches()
    t = timed(lambda: msa.msa_topk_rows(s, k, idx))
    launches = (msa.msa_kernel_launches() - l0) * steps // (steps + warmup)
    nbytes = rows * n * 4 + rows * k * 4
    gbs = nbytes / t / 1e9
    traffic, tnote = captured_traffic("topk_rows", rows / CAPTURES["topk_rows"]["rows"]) \
        if "topk_rows" in CAPTURES else (None, "no capture recorded")
    del s
    return {"workload": f"topk_rows_{rows}x1024_k15", "metric": "exp-free top-k rows/s (k = 15 of 1,024 fp32)",
            "value": rows / t, "unit": "rows/s", "ms": t * 1e3, "gpu_launches": int(launches),
            "torch_topk_ms": None if t_ref is None else t_ref * 1e3,
            "speedup_vs_torch_topk": None if t_ref is None else t_ref / t,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": traffic, "traffic_note": tnote,
                         "kernel": "topk_rows_kernel",
                         "algorithmic": f"{nbytes} B per launch (scores read once, ids written)",
                         "peak_source": f"{peak_src} copy"}}


def e2e_pipelined(torch, pipeline, x, pbufs, ds, dbufs, graph, steps, warmup, dev):
    """The step end to end through the public API with host buffers: every step copies its
    prefill inputs and its decode-token inputs from pinned host memory, runs the prefill pass and
    the decode step, and copies the prefill output and the decode output back. Copies of step
    i + 1's inputs and of step i - 1's outputs run on their own streams (one per direction)
    while step i computes; inputs and outputs are double-buffered on the device. Time = first
    input copy to last output copy, divided by the steps."""
    names = list(x.keys())
    host_in = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in x.items()}
    for k in names:
        host_in[k].copy_(x[k])
    dev_in = [{k: torch.empty_like(v) for k, v in x.items()} for _ in range(2)]
    outs = [pbufs["out"], torch.empty_like(pbufs["out"])]
    host_out = [torch.empty(pbufs["out"].shape, dtype=pbufs["out"].dtype, pin_memory=True) for _ in range(2)]
    dnames = ("q", "q_idx", "k_idx_new", "k_new", "v_new")
    dhost = {k: torch.empty(ds[k].shape, dtype=ds[k].dtype, pin_memory=True) for k in dnames}
    for k in dnames:
        dhost[k].copy_(ds[k])
    dhost_out = [torch.empty(dbufs["out"].shape, dtype=dbufs["out"].dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values()) + \
        sum(v.numel() * v.element_size() for v in dhost.values())
    d2h = host_out[0].numel() * host_out[0].element_size() + dhost_out[0].numel() * dhost_out[0].element_size()
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def run(n):
        in_ready, comp_done, out_done = [], [], []
        start = ev()
        start.record(s_in)
        for i in range(n):
            buf = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])          # the compute that read dev_in[buf] is done
                for k in names:
                    dev_in[buf][k].copy_(host_in[k], non_blocking=True)
                e = ev()
                e.record(s_in)
                in_ready.append(e)
            comp.wait_event(in_ready[i])
            if i >= 2:
                comp.wait_event(out_done[i - 2])               # outs[buf] has been copied out
            d = dev_in[buf]
            bufs = dict(pbufs, out=outs[buf])
            pipeline.prefill(d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], bufs, comp)
            for k in dnames:
                ds[k].copy_(dhost[k], non_blocking=True)
            graph.replay()
            e = ev()
            e.record(comp)
            comp_done.append(e)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                host_out[buf].copy_(outs[buf], non_blocking=True)
                dhost_out[buf].copy_(dbufs["out"], non_blocking=True)
                e = ev()
                e.record(s_out)
                out_done.append(e)
        end = ev()
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end) * 1e-3 / n

    run(max(2, warmup))
    t = run(steps)
    return t, int(h2d), int(d2h)


def run_ours(args):
    import torch
    import torch.distributed as dist
    import block_sparse_gqa_branch_b200 as msa
    from block_sparse_gqa_branch_b200 import pipeline

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    msa.load()

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, dev)

    wp, wd = workloads(args)
    do_prefill, do_decode = args.only in (None, "prefill", "index"), args.only in (None, "decode")
    do_main = args.only in (None, "prefill")
    x = synth.prefill_inputs_torch(wp, dev) if do_prefill else None
    if do_prefill and not do_main:                 # index branch alone: its inputs only
        x = {"q_idx": x["q_idx"], "k_idx": x["k_idx"]}
        torch.cuda.empty_cache()
    pbufs = pipeline.prefill_buffers(wp.B, wp.N, wp.Hq, wp.G, dev, with_main=do_main) if do_prefill else None
    ds = build_decode_state(wd, dev) if do_decode else None
    dbufs = pipeline.decode_buffers(wd.B, wd.Hq, wd.G, max(wd.ctx), dev) if do_decode else None
    flush_l2 = make_flusher(torch, dev)
    stream = torch.cuda.current_stream()

    def decode_call():
        pipeline.decode_step(ds["q"], ds["q_idx"], ds["k_idx_new"], ds["k_new"], ds["v_new"], ds["ctx"],
                             ds["k_cache"], ds["v_cache"], ds["tail"], ds["pooled"], dbufs)

    # eager warm-up (sets kernel attributes), then capture the decode step in a CUDA graph
    graph = None
    if do_prefill:
        pipeline.prefill_index(x["q_idx"], x["k_idx"], pbufs)
    if do_main:
        pipeline.prefill_main(x["q"], x["k"], x["v"], pbufs)
    if do_decode:
        decode_call()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            decode_call()
    torch.cuda.synchronize()

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    t_index, t_main, t_dec = [], [], []

    def one_step(record: bool):
        flush_l2()
        e0, e1, e2, e3, e4 = ev(), ev(), ev(), ev(), ev()
        e0.record(stream)
        if do_prefill:
            pipeline.prefill_index(x["q_idx"], x["k_idx"], pbufs)
        e1.record(stream)
        if do_main:
            pipeline.prefill_main(x["q"], x["k"], x["v"], pbufs)
        e2.record(stream)
        flush_l2()
        e3.record(stream)
        if do_decode:
            graph.replay()
        e4.record(stream)
        return (e0, e1, e2, e3, e4) if record else None

    for _ in range(args.warmup):
        one_step(False)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    launches_before = msa.msa_kernel_launches()
    msa.msa_kernel_timing_read(0)
    msa.msa_kernel_timing_enable(True)            # events around each eager kernel launch
    with ClockSampler(local) as clk:
        evs = [one_step(True) for _ in range(args.steps)]
        torch.cuda.synchronize()
    msa.msa_kernel_timing_enable(False)
    kernels = kernel_means(msa.msa_kernel_timing_read(), args.steps)
    kernels = {k: {"ms": max_over_ranks(kernels[k]["ms"]), "launches": kernels[k]["launches"]} for k in sorted(kernels)}
    barrier()
    torch.cuda.synchronize()
    launches_eager = msa.msa_kernel_launches() - launches_before
    for e0, e1, e2, e3, e4 in evs:
        t_index.append(e0.elapsed_time(e1) * 1e-3)
        t_main.append(e1.elapsed_time(e2) * 1e-3)
        t_dec.append(e3.elapsed_time(e4) * 1e-3)
    decode_graph_kernels = 3 if do_decode else 0
    gpu_launches = launches_eager + decode_graph_kernels * args.steps

    # check the device error words after the timed region
    for key in (("ws_select", "ws_attn") if do_main else ("ws_select",) if do_prefill else ()):
        st_, info = msa.msa_get_device_status(pbufs[key])
        if st_ != 0:
            raise SystemExit(f"device status {st_} in prefill {key}: {info}")
    for key in (("ws_append", "ws_select", "ws_attn") if do_decode else ()):
        st_, info = msa.msa_get_device_status(dbufs[key])
        if st_ != 0:
            raise SystemExit(f"device status {st_} in decode {key}: {info}")

    tp = max_over_ranks(statistics.mean([a + b for a, b in zip(t_index, t_main)]))
    tmain = max_over_ranks(statistics.mean(t_main))
    tidx = max_over_ranks(statistics.mean(t_index))
    tdec = max_over_ranks(statistics.mean(t_dec))
    peaks, peak_src = load_peaks()
    pre = None
    if do_main:
        pre = prefill_report(wp, [tidx], [tmain], peaks, peak_src, world, launches_eager, kernels)
    dec = decode_report(wd, [tdec], peaks, peak_src, decode_graph_kernels * args.steps,
                        traffic_name="decode_step",
                        scale=(decode_step_bytes(wd)["total"] / CAPTURES["decode_step"]["algorithmic_bytes"]
                               if "decode_step" in CAPTURES else 1.0))

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e and do_prefill and do_decode:
        te, h2d, d2h = e2e_pipelined(torch, pipeline, x, pbufs, ds, dbufs, graph, args.steps, args.warmup, dev)
        te = max_over_ranks(te)
        e2e = {"value": wp.N * wp.B * world / te, "unit": "tok/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": te * 1e3,
               "note": "through the public API: prefill inputs and decode-token inputs copied from pinned host "
                       "memory and the prefill and decode outputs copied back every step; copies of the next "
                       "step's inputs and the previous step's outputs overlap this step's compute (one stream "
                       "per direction, double-buffered); value counts prefill tokens"}

    # ---------------------------------------------------------------- the other workloads
    extra = {}
    if not args.no_extra and args.only is None and not (args.prefill_tokens or args.decode_batch):
        graph = None
        del x, pbufs, ds, dbufs
        torch.cuda.empty_cache()
        n_x, w_x = min(args.steps, 10), 3
        ti2, tm2, l2, k2 = time_prefill(torch, PREFILL_32K, dev, n_x, w_x, flush_l2)
        k2 = {k: {"ms": max_over_ranks(k2[k]["ms"]), "launches": k2[k]["launches"]} for k in sorted(k2)}
        r = prefill_report(PREFILL_32K, [max_over_ranks(statistics.mean(ti2))], [max_over_ranks(statistics.mean(tm2))],
                           peaks, peak_src, world, l2, k2)
        extra[PREFILL_32K.name] = r
        torch.cuda.empty_cache()
        # the small prefill (4,096 tokens, 4 query heads / 1 group): launch-bound, L2-resident
        ti4, tm4, l4, k4 = time_prefill(torch, PREFILL_4K, dev, n_x, w_x, flush_l2)
        k4 = {k: {"ms": max_over_ranks(k4[k]["ms"]), "launches": k4[k]["launches"]} for k in sorted(k4)}
        extra[PREFILL_4K.name] = prefill_report(PREFILL_4K, [max_over_ranks(statistics.mean(ti4))],
                                                [max_over_ranks(statistics.mean(tm4))], peaks, peak_src, world, l4, k4)
        torch.cuda.empty_cache()
        td5, l5 = time_decode(torch, DECODE_1M, dev, n_x, w_x, flush_l2)
        extra[DECODE_1M.name] = decode_report(
            DECODE_1M, [max_over_ranks(statistics.mean(td5))], peaks, peak_src, l5, traffic_name="decode_step",
            scale=(decode_step_bytes(DECODE_1M)["total"] / CAPTURES["decode_step"]["algorithmic_bytes"]
                   if "decode_step" in CAPTURES else 1.0))
        torch.cuda.empty_cache()
        td8, l8 = time_decode(torch, DECODE, dev, n_x, w_x, flush_l2, fp8=True)
        r8 = decode_report(DECODE, [max_over_ranks(statistics.mean(td8))], peaks, peak_src, l8, fp8=True)
        r8["workload"] = DECODE.name + "_fp8kv"
        extra[r8["workload"]] = r8
        torch.cuda.empty_cache()
        tb = max_over_ranks(statistics.mean(time_backward(torch, PREFILL_32K, dev, n_x, w_x, flush_l2)))
        bflops = 2.5 * prefill_main_flops(PREFILL_32K)          # S, dP, dV, dK, dQ: five products
        extra[PREFILL_32K.name + "_backward"] = {
            "workload": PREFILL_32K.name + "_backward", "backward_ms": tb * 1e3,
            "value": PREFILL_32K.N * PREFILL_32K.B * world / tb, "unit": "tok/s",
            "roofline": {"bound": "tensor", "achieved": bflops / tb / 1e12, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": bflops / tb / 1e12 / peaks["bf16_tflops"], "traffic": None,
                         "kernel": "main-branch backward (msa_sparse_attn_prefill_backward: inverted index, D, dQ/dK/dV)",
                         "algorithmic": f"{bflops:.4e} FLOP per launch (10 x 128 per attended head-key pair)",
                         "peak_source": f"{peak_src} burst bf16"}}
        torch.cuda.empty_cache()
        tc, nchunks = time_prefill_chunked(torch, PREFILL, dev, 16384, n_x, w_x, flush_l2)
        tc = max_over_ranks(statistics.mean(tc))
        cflops = prefill_main_flops(PREFILL)
        extra[PREFILL.name + "_chunked16k"] = {
            "workload": PREFILL.name + f" in {nchunks} chunks of 16,384 tokens", "prefill_ms": tc * 1e3,
            "value": PREFILL.N * PREFILL.B * world / tc, "unit": "tok/s",
            "roofline": {"bound": "tensor", "achieved": cflops / tc / 1e12, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": cflops / tc / 1e12 / peaks["bf16_tflops"], "traffic": None,
                         "kernel": "chunked prefill, all chunks (pooling, selection and main branch per chunk)",
                         "algorithmic": f"{cflops:.4e} main-branch FLOP per pass", "peak_source": f"{peak_src} burst bf16"}}
        torch.cuda.empty_cache()
        tk = topk_report(torch, dev, n_x, w_x, peaks, peak_src)
        tk["ms"] = max_over_ranks(tk["ms"])
        tk["value"] = 8 * 131072 * world / (tk["ms"] * 1e-3)
        extra[tk["workload"]] = tk
        torch.cuda.empty_cache()

    if world > 1:
        graph = None
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = cpu_dec = None
    if not args.no_cpu_baseline and args.only is None:
        try:
            cpu = cpu_baseline(wp, budget_s=args.cpu_budget)
        except Exception as exc:  # reported, never fatal for the GPU number
            cpu = {"value": None, "unit": "tok/s", "cores": os.cpu_count(), "kind": "oracle",
                   "sample": f"failed: {exc!r}"}
        try:
            cpu_dec = {DECODE.name: cpu_baseline_decode(DECODE)}
            if not args.no_extra:
                cpu_dec[DECODE_1M.name] = cpu_baseline_decode(DECODE_1M)
        except Exception as exc:
            cpu_dec = {"failed": repr(exc)}
    clocks = clk.summary()
    line = {
        "metric": METRIC,
        "value": wp.N * wp.B * world / tp,
        "unit": "tok/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": (tp + tdec) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64 -> N(0,1) quantiles -> bf16), generated on the device",
        "config": config_block(wp, wd),
        "prefill_ms": tp * 1e3,
        "prefill_index_ms": tidx * 1e3,
        "prefill_main_ms": tmain * 1e3,
        "decode_step_us": tdec * 1e6,
        "roofline": pre["roofline"] if pre is not None else None,
        "roofline_call": pre["roofline_call"] if pre is not None else None,
        "prefill_kernels_ms": pre["kernels_ms"] if pre is not None else None,
        "prefill_hbm": pre["hbm"] if pre is not None else None,
        "roofline_index": pre["roofline_index"] if pre is not None else None,
        "roofline_decode": dec["roofline"] if do_decode else None,
        "clocks": clocks,
        "gpu_launches": int(gpu_launches),
        "e2e": e2e,
        "cpu_baseline": cpu,
        "cpu_baseline_decode": cpu_dec,
        "workloads": extra,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_topk(args):
    """The exp-free top-k micro-benchmark alone (one GPU), as one JSON line."""
    import torch
    import block_sparse_gqa_branch_b200 as msa
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    msa.load()
    peaks, peak_src = load_peaks()
    with ClockSampler(local) as clk:
        r = topk_report(torch, dev, args.steps, args.warmup, peaks, peak_src, rows=args.topk_rows)
    line = {"metric": r["metric"], "value": r["value"], "unit": r["unit"], "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded normal scores generated on the device)",
            "config": {"workload": r["workload"], "rows": args.topk_rows, "n": 1024, "k": 15,
                       "l2": "inputs (4.3 GB) larger than L2, no flush"},
            "roofline": r["roofline"], "torch_topk_ms": r["torch_topk_ms"],
            "speedup_vs_torch_topk": r["speedup_vs_torch_topk"], "clocks": clk.summary(),
            "gpu_launches": r["gpu_launches"]}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads (32K planted prefill, 1M ragged decode, top-k)")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle CPU time")
    ap.add_argument("--only", choices=["prefill", "index", "decode"], default=None,
                    help="run one half of the step (profiler captures; not a benchmark value)")
    ap.add_argument("--prefill-tokens", type=int, default=0, help="smaller prefill for profiler captures")
    ap.add_argument("--decode-batch", type=int, default=0, help="smaller decode batch for profiler captures")
    ap.add_argument("--topk-rows", type=int, default=8 * 131072, help="rows of the top-k benchmark (captures)")
    ap.add_argument("--topk", action="store_true",
                    help="the exp-free top-k micro-benchmark against torch.topk instead of the step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.topk:
        return run_topk(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
