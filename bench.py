#!/usr/bin/env python
"""Benchmark of the MSA (MiniMax Sparse Attention over GQA) hot path on B200.

One step = one pass of the whole hot path on synthetic inputs already resident in HBM:
  * prefill of 131,072 tokens, batch 1, 64 query heads / 8 KV groups (pooling, block scoring +
    exp-free top-16 selection, main-branch sparse attention), and
  * one decode step of a batch of 16 sequences at 131,072 cached tokens (append + pooled-key
    update, selection, attention split over the selected blocks), replayed from a CUDA graph.
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
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum, one ncu capture) of one decode
# step of batch 16 at 131,072 tokens: select_decode_kernel 8,430,080 B read and
# attn_decode_kernel 32,116,736 B read + 11,264 B written, captured at batch 4 (same contexts),
# times 4 (both kernels' work is per (sequence, group)); the append kernel's few KB are left
# out. Re-capture when those kernels change.
DECODE_STEP_DRAM_BYTES = 4 * (8_430_080 + 32_116_736 + 11_264)


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
    Returns seconds per token (all G groups), including the group's pooling."""
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


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    cache = {}
    n = 64
    _, el = oracle_prefill_sample(PREFILL, n, 0, cache=cache)
    n_step = int(max(32, min(20000, n * 8.0 / max(el, 1e-3))))
    times = []
    for s in range(args.warmup + args.steps):
        per_tok, el = oracle_prefill_sample(PREFILL, n_step, 0, seed=100 + s, cache=cache)
        if s >= args.warmup:
            times.append(per_tok)
    per_tok = statistics.mean(times)
    value = 1.0 / per_tok
    sample = (f"each step: {n_step} (token, group 0) rows of {PREFILL.name} drawn uniformly, "
              f"selection + attention, plus group 0's pooling, scaled to whole tokens (x{PREFILL.G})")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_tok * PREFILL.N * 1e3,
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
    do_prefill, do_decode = args.only in (None, "prefill"), args.only in (None, "decode")
    x = synth.prefill_inputs_torch(wp, dev)
    pbufs = pipeline.prefill_buffers(wp.B, wp.N, wp.Hq, wp.G, dev)
    ds = build_decode_state(wd, dev) if do_decode else None
    dbufs = pipeline.decode_buffers(wd.B, wd.Hq, wd.G, max(wd.ctx), dev) if do_decode else None
    # L2 flush between timed steps: write a buffer larger than L2 (126 MB), then read another
    # one, so that the written lines are written back before the timed region (a write alone
    # leaves ~126 MB of dirty lines whose write-back would land inside the next step)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        flush_rd.sum()
    stream = torch.cuda.current_stream()

    def decode_call():
        pipeline.decode_step(ds["q"], ds["q_idx"], ds["k_idx_new"], ds["k_new"], ds["v_new"], ds["ctx"],
                             ds["k_cache"], ds["v_cache"], ds["tail"], ds["pooled"], dbufs)

    # eager warm-up (sets kernel attributes), then capture the decode step in a CUDA graph
    graph = None
    if do_prefill:
        pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], pbufs)
    if do_decode:
        decode_call()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            decode_call()
    torch.cuda.synchronize()

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    t_index, t_main, t_dec = [], [], []
    launches0 = msa.msa_kernel_launches()

    def one_step(record: bool):
        flush_l2()
        e0, e1, e2, e3, e4 = ev(), ev(), ev(), ev(), ev()
        e0.record(stream)
        if do_prefill:
            pipeline.prefill_index(x["q_idx"], x["k_idx"], pbufs)
        e1.record(stream)
        if do_prefill:
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
    with ClockSampler(local) as clk:
        evs = [one_step(True) for _ in range(args.steps)]
        torch.cuda.synchronize()
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
    for key in ("ws_select", "ws_attn"):
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
    flops = prefill_main_flops(wp)
    achieved_tf = flops / tmain / 1e12
    dbytes = decode_step_bytes(wd)
    dec_gbs = dbytes["total"] / tdec / 1e9

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e and do_prefill and do_decode:
        host_in = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in x.items()}
        for k in x:
            host_in[k].copy_(x[k])
        dev_in = {k: torch.empty_like(v) for k, v in x.items()}
        host_out = torch.empty(pbufs["out"].shape, dtype=pbufs["out"].dtype, pin_memory=True)
        dnames = ("q", "q_idx", "k_idx_new", "k_new", "v_new")
        dhost = {k: torch.empty(ds[k].shape, dtype=ds[k].dtype, pin_memory=True) for k in dnames}
        for k in dnames:
            dhost[k].copy_(ds[k])
        dhost_out = torch.empty(dbufs["out"].shape, dtype=dbufs["out"].dtype, pin_memory=True)
        h2d = sum(v.numel() * v.element_size() for v in host_in.values()) + \
            sum(v.numel() * v.element_size() for v in dhost.values())
        d2h = host_out.numel() * host_out.element_size() + dhost_out.numel() * dhost_out.element_size()
        times = []
        for s in range(max(1, args.warmup // 2) + args.steps):
            flush_l2()
            torch.cuda.synchronize()
            e0, e1 = ev(), ev()
            e0.record(stream)
            for k in x:
                dev_in[k].copy_(host_in[k], non_blocking=True)
            pipeline.prefill(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["q_idx"], dev_in["k_idx"], pbufs)
            host_out.copy_(pbufs["out"], non_blocking=True)
            for k in dnames:
                ds[k].copy_(dhost[k], non_blocking=True)
            graph.replay()
            dhost_out.copy_(dbufs["out"], non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if s >= max(1, args.warmup // 2):
                times.append(e0.elapsed_time(e1) * 1e-3)
        te = max_over_ranks(statistics.mean(times))
        e2e = {"value": wp.N * wp.B * world / te, "unit": "tok/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": te * 1e3,
               "note": "prefill inputs and decode-token inputs copied from pinned host memory, prefill output "
                       "and decode output copied back, every step; value counts prefill tokens"}

    if world > 1:
        graph = None
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = None
    if not args.no_cpu_baseline and args.only is None:
        try:
            cpu = cpu_baseline(wp, budget_s=args.cpu_budget)
        except Exception as exc:  # reported, never fatal for the GPU number
            cpu = {"value": None, "unit": "tok/s", "cores": os.cpu_count(), "kind": "oracle",
                   "sample": f"failed: {exc!r}"}
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
        "roofline": ({"bound": "tensor", "achieved": achieved_tf, "peak": peaks["bf16_tflops"],
                      "unit": "TFLOP/s", "frac": achieved_tf / peaks["bf16_tflops"], "traffic": None,
                      "kernel": "prefill main branch (msa_sparse_attn_prefill, all its kernels)",
                      "algorithmic": f"{flops:.4e} FLOP per launch", "peak_source": f"{peak_src} burst bf16"}
                     if do_prefill else None),
        "roofline_decode": ({"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": dec_gbs / peaks["hbm_gbs"],
                             "traffic": DECODE_STEP_DRAM_BYTES if (wd.B, wd.ctx) == (16, (131072,) * 16) else None,
                             "kernel": "decode step (append + select + attention, one graph replay)",
                             "algorithmic": f"{dbytes['total']} B per step", "peak_source": f"{peak_src} copy"}
                            if do_decode else None),
        "clocks": clocks,
        "gpu_launches": int(gpu_launches),
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_topk(args):
    """Exp-free top-k micro-benchmark (one GPU): msa_topk_rows against torch.topk on the block
    scores of 8 groups at 131,072 tokens, [1,048,576, 1024] fp32 with k = 15 (the fully-past
    blocks a query keeps besides its own). The scores are seeded normal values generated on the
    device; at 4.3 GB they are larger than L2, so no flush is needed between iterations."""
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
    rows, n, k = 8 * 131072, 1024, 15
    s = torch.randn(rows, n, device=dev, generator=torch.Generator(device=dev).manual_seed(0x4D5341))
    idx = torch.empty(rows, k, dtype=torch.int32, device=dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3)
        return statistics.median(ts)

    t_ref = timed(lambda: torch.topk(s, k, dim=1))
    launches0 = msa.msa_kernel_launches()
    with ClockSampler(local) as clk:
        t = timed(lambda: msa.msa_topk_rows(s, k, idx))
    launches = msa.msa_kernel_launches() - launches0
    peaks, peak_src = load_peaks()
    nbytes = rows * n * 4 + rows * k * 4
    gbs = nbytes / t / 1e9
    line = {
        "metric": "exp-free top-k rows/s (k = 15 of 1,024 fp32 block scores per row)",
        "value": rows / t, "unit": "rows/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (seeded normal scores generated on the device)",
        "config": {"workload": "topk_rows_1048576x1024_k15", "rows": rows, "n": n, "k": k,
                   "l2": "inputs (4.3 GB) larger than L2, no flush"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None, "kernel": "topk_rows_kernel",
                     "algorithmic": f"{nbytes} B per launch (scores read once, ids written)",
                     "peak_source": f"{peak_src} copy"},
        "torch_topk_ms": t_ref * 1e3, "speedup_vs_torch_topk": t_ref / t,
        "clocks": clk.summary(), "gpu_launches": int(launches),
    }
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
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle CPU time")
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="run one half of the step (profiler captures; not a benchmark value)")
    ap.add_argument("--prefill-tokens", type=int, default=0, help="smaller prefill for profiler captures")
    ap.add_argument("--decode-batch", type=int, default=0, help="smaller decode batch for profiler captures")
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
