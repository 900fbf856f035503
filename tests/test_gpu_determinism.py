"""Run-to-run determinism of the GPU path, through the C ABI: the check that stands in for a
race detector. A data race in a kernel (a missing barrier, a buffer reused too early) shows
up as results that change between identical calls.

* prefill: three eager calls and three replays of a CUDA graph of the whole pass give the same
  selection and bit-identical outputs and lse (every partial row is computed by one CTA, and
  the merge of a query's partials runs in a fixed slot order, so nothing depends on timing);
* decode: the selection is identical over three calls and three graph replays; the output
  may differ in rounding only, because a group split over CTAs is merged by whichever CTA
  arrives last (an atomic decides the order of the fp32 merge).
"""
import numpy as np
import pytest
import torch

import synth
from block_sparse_gqa_branch_b200 import msa_get_device_status, msa_index_select, msa_sparse_attn_decode, pipeline
from tests.test_gpu_decode import build_decode_state

pytestmark = pytest.mark.gpu


def test_prefill_is_deterministic_eager_and_graph(cuda_ok):
    w = synth.Workload(name="det", kind="prefill", B=1, N=20000 + 77, Hq=64, G=8, seed=31337)
    x = synth.prefill_inputs_torch(w, "cuda")
    bufs = pipeline.prefill_buffers(w.B, w.N, w.Hq, w.G, "cuda")

    def run():
        pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], bufs)

    results = []
    for _ in range(3):
        run()
        torch.cuda.synchronize()
        results.append((bufs["sel"].clone(), bufs["out"].clone(), bufs["lse"].clone()))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(3):
        bufs["out"].zero_()
        bufs["sel"].fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        results.append((bufs["sel"].clone(), bufs["out"].clone(), bufs["lse"].clone()))
    for key in ("ws_select", "ws_attn"):
        assert msa_get_device_status(bufs[key])[0] == 0
    s0, o0, l0 = results[0]
    for i, (s, o, l) in enumerate(results[1:], 1):
        assert torch.equal(s, s0), f"selection differs in run {i}"
        assert torch.equal(o.view(torch.int16), o0.view(torch.int16)), f"output bits differ in run {i}"
        assert torch.equal(l.view(torch.int32), l0.view(torch.int32)), f"lse bits differ in run {i}"


def test_decode_selection_is_deterministic_eager_and_graph(cuda_ok):
    ctx = (70000, 3000, 129, 50000)
    w = synth.Workload(name="det", kind="decode", B=len(ctx), Hq=64, G=8, ctx=ctx, seed=777)
    l_cap = (max(ctx) + 1 + 127) // 128 * 128 + 128
    st = build_decode_state(w, l_cap, garbage=False)
    bufs = pipeline.decode_buffers(w.B, w.Hq, w.G, max(ctx), "cuda")
    # the new tokens go in first (append is not idempotent in general, so it runs once)
    pipeline.decode_step(st["q"], st["q_idx"], st["k_idx_new"], st["k_new"], st["v_new"], st["ctx"],
                         st["k_cache"], st["v_cache"], st["tail"], st["pooled"], bufs)
    s, mp = bufs["shape"], bufs["max_pos"]
    nb_cap = st["pooled"].shape[2]

    def run():
        msa_index_select(s, st["q_idx"], 1, st["ctx"], mp, st["pooled"], nb_cap, bufs["sel"], bufs["ws_select"])
        msa_sparse_attn_decode(s, st["q"], st["k_cache"], st["v_cache"], l_cap, st["ctx"], mp, bufs["sel"],
                               bufs["out"], bufs["lse"], bufs["ws_attn"])

    results = []
    for _ in range(3):
        run()
        torch.cuda.synchronize()
        results.append((bufs["sel"].clone(), bufs["out"].float().clone()))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(3):
        bufs["sel"].fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        results.append((bufs["sel"].clone(), bufs["out"].float().clone()))
    for key in ("ws_append", "ws_select", "ws_attn"):
        assert msa_get_device_status(bufs[key])[0] == 0
    s0, o0 = results[0]
    for i, (sel, o) in enumerate(results[1:], 1):
        assert torch.equal(sel, s0), f"selection differs in run {i}"
        # rounding only: one bf16 step of the value at most
        tol = o0.abs() * 2.0 ** -7 + 1e-6
        assert bool(((o - o0).abs() <= tol).all()), f"output differs beyond rounding in run {i}"
    assert np.isfinite(o0.cpu().numpy()).all()
