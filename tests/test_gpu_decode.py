"""GPU parity of the decode step (append, select, split-KV attention) against the fp64 oracle,
through the C ABI, plus the cross-path checks decode(L) == prefill row L and 128 appends ==
block pooling."""
import numpy as np
import pytest
import torch

import oracle
import synth
from block_sparse_gqa_branch_b200 import (Shape, msa_get_device_status, msa_index_select,
                                          msa_pool_index_keys, msa_pooled_keys_append, msa_sparse_attn_decode,
                                          pipeline)
from tests.gpu_util import check_selection, dev_bf16, f32, host_bits
from tests.msa_check import assert_close_attention

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC0


def build_decode_state(w, l_cap, garbage=True):
    """Caches holding positions 0..L_b-1 of every sequence (the new token is appended by the
    step), pooled keys built by the library's pooling kernel, plus the step's inputs."""
    B, G = w.B, w.G
    dev = "cuda"
    k_cache = torch.empty(B, G, l_cap, 128, dtype=torch.bfloat16, device=dev)
    v_cache = torch.empty_like(k_cache)
    if garbage:       # positions past the context hold NaNs: they must never reach the output
        k_cache.view(torch.int16).fill_(NAN_BF16)
        v_cache.view(torch.int16).fill_(NAN_BF16)
    nb_cap = l_cap // 128 + 1
    pooled = torch.full((B, G, nb_cap, 64), float("nan"), device=dev)
    tail = torch.zeros(B, G, 64, device=dev)
    q = torch.empty(B, w.Hq, 128, dtype=torch.bfloat16, device=dev)
    q_idx = torch.empty(B, G, 64, dtype=torch.bfloat16, device=dev)
    k_idx_new = torch.empty(B, G, 64, dtype=torch.bfloat16, device=dev)
    k_new = torch.empty(B, G, 128, dtype=torch.bfloat16, device=dev)
    v_new = torch.empty_like(k_new)
    for b in range(B):
        Lb = w.ctx[b]
        kk = synth.decode_seq_torch(w, b, "k", dev)           # [G, L, d]
        vv = synth.decode_seq_torch(w, b, "v", dev)
        ki = synth.decode_seq_torch(w, b, "k_idx", dev)       # [L, G, dI]
        k_cache[b, :, :Lb] = kk[:, :Lb]
        v_cache[b, :, :Lb] = vv[:, :Lb]
        k_new[b], v_new[b], k_idx_new[b] = kk[:, Lb], vv[:, Lb], ki[Lb]
        q[b] = synth.decode_seq_torch(w, b, "q", dev)
        q_idx[b] = synth.decode_seq_torch(w, b, "q_idx", dev)
        if Lb > 0:
            msa_pool_index_keys(Shape.make(1, w.Hq, G), ki[:Lb].contiguous(), Lb, pooled[b], nb_cap, tail[b])
    ctx = torch.tensor(list(w.ctx), dtype=torch.int32, device=dev)
    return dict(k_cache=k_cache, v_cache=v_cache, pooled=pooled, tail=tail, q=q, q_idx=q_idx,
                k_idx_new=k_idx_new, k_new=k_new, v_new=v_new, ctx=ctx, nb_cap=nb_cap)


def run_step(w, st):
    bufs = pipeline.decode_buffers(w.B, w.Hq, w.G, max(w.ctx), "cuda")
    out, lse, sel = pipeline.decode_step(st["q"], st["q_idx"], st["k_idx_new"], st["k_new"], st["v_new"],
                                         st["ctx"], st["k_cache"], st["v_cache"], st["tail"], st["pooled"], bufs)
    torch.cuda.synchronize()
    for key in ("ws_append", "ws_select", "ws_attn"):
        s, info = msa_get_device_status(bufs[key])
        assert s == 0, (key, s, info)
    return f32(host_bits(out)), lse.cpu().numpy(), sel.cpu().numpy()


def oracle_decode(w, sel_gpu):
    """Oracle selection and attention (on the GPU's selection) for every (sequence, group)."""
    res = []
    for b in range(w.B):
        Lb = w.ctx[b]
        ki = synth.decode_seq_np(w, b, "k_idx")               # [L, G, dI]
        pooled, _ = oracle.pool(ki, 128)
        qi = synth.decode_seq_np(w, b, "q_idx")
        q = synth.decode_seq_np(w, b, "q")
        kk = synth.decode_seq_np(w, b, "k")
        vv = synth.decode_seq_np(w, b, "v")
        for g in range(w.G):
            t = np.array([Lb])
            s, kth, _ = oracle.select_rows(t, qi[g][None], pooled[g])
            o, lse, nk = oracle.attend_rows(t, q[None, g * w.Hg:(g + 1) * w.Hg], kk[g], vv[g], sel_gpu[b, g][None])
            res.append(dict(b=b, g=g, sel=s[0], kth=kth[0], o=o[0], lse=lse[0], pooled=pooled[g], qi=qi[g], t=t))
    return res


@pytest.mark.parametrize("ctx,Hq,G", [((4999, 2048, 127, 255), 16, 2), ((20000,), 64, 8), ((1, 0, 128 * 17), 8, 1),
                                      ((3000, 70), 4, 4), ((3000, 129), 8, 4), ((2500, 40), 16, 4),
                                      ((2900, 1), 16, 1)])
def test_decode_step_matches_oracle(cuda_ok, ctx, Hq, G):
    w = synth.Workload(name="t", kind="decode", B=len(ctx), Hq=Hq, G=G, ctx=tuple(ctx), seed=4242 + sum(ctx))
    l_cap = (max(ctx) + 1 + 127) // 128 * 128 + 128
    st = build_decode_state(w, l_cap)
    out, lse, sel = run_step(w, st)
    ref = oracle_decode(w, sel)
    for r in ref:
        b, g = r["b"], r["g"]
        check_selection(sel[b, g][None], r["sel"][None], np.array([r["kth"]]), r["qi"][None], r["pooled"], r["t"],
                        label=f"decode ctx={ctx} Hq={Hq} G={G}")
        assert_close_attention(out[b, g * w.Hg:(g + 1) * w.Hg], r["o"], f"decode b={b} g={g}")
        np.testing.assert_allclose(lse[b, g * w.Hg:(g + 1) * w.Hg], r["lse"], rtol=0, atol=2e-3)
    # the appended token and the block it closed
    for b in range(w.B):
        Lb = w.ctx[b]
        kk = synth.decode_seq_np(w, b, "k")
        assert (host_bits(st["k_cache"][b, :, Lb]) == kk[:, Lb]).all()
        if (Lb + 1) % 128 == 0:
            ki = synth.decode_seq_np(w, b, "k_idx")
            ref_pool, _ = oracle.pool(ki, 128)
            got = st["pooled"][b, :, Lb // 128].cpu().numpy()
            np.testing.assert_allclose(got, ref_pool[:, Lb // 128], rtol=1e-5, atol=1e-6)


def test_decode_is_last_prefill_row(cuda_ok):
    L = 128 * 19 + 37
    wp = synth.Workload(name="p", kind="prefill", B=1, N=L + 1, Hq=16, G=2, seed=91)
    x = synth.prefill_inputs_np(wp)
    d = {k: dev_bf16(v) for k, v in x.items()}
    bufs = pipeline.prefill_buffers(1, L + 1, 16, 2, "cuda")
    out_p, lse_p, sel_p = pipeline.prefill(d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], bufs)
    # decode state from the same tensors: cache = first L tokens, the step appends token L
    l_cap = L + 129
    kc = torch.zeros(1, 2, l_cap, 128, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kc[:, :, :L] = d["k"][:, :, :L]
    vc[:, :, :L] = d["v"][:, :, :L]
    nb_cap = l_cap // 128 + 1
    pooled = torch.zeros(1, 2, nb_cap, 64, device="cuda")
    tail = torch.zeros(1, 2, 64, device="cuda")
    shape = Shape.make(1, 16, 2)
    msa_pool_index_keys(shape, d["k_idx"][:, :L].contiguous(), L, pooled, nb_cap, tail)
    ctx = torch.tensor([L], dtype=torch.int32, device="cuda")
    dbufs = pipeline.decode_buffers(1, 16, 2, L, "cuda")
    out_d, lse_d, sel_d = pipeline.decode_step(d["q"][:, L].contiguous(), d["q_idx"][:, L].contiguous(),
                                               d["k_idx"][:, L].contiguous(), d["k"][:, :, L].contiguous(),
                                               d["v"][:, :, L].contiguous(), ctx, kc, vc, tail, pooled, dbufs)
    torch.cuda.synchronize()
    # The two paths score in different fp32 orders (fma chains vs tensor-core sums), so their
    # sets may differ only where the oracle's fp64 scores make a near-tie; both must be valid.
    pooled_o, _ = oracle.pool(x["k_idx"][0, :L], 128)
    t = np.array([L])
    sd, sp = sel_d[0].cpu().numpy(), sel_p[0, L].cpu().numpy()
    for g in range(2):
        qi = x["q_idx"][0, L, g][None]
        ref, kth, _ = oracle.select_rows(t, qi, pooled_o[g])
        check_selection(sd[g][None], ref, kth, qi, pooled_o[g], t, label="decode(L) vs prefill row L: decode")
        check_selection(sp[g][None], ref, kth, qi, pooled_o[g], t, label="decode(L) vs prefill row L: prefill")
    same = (sd == sp).all(axis=1)
    assert same.any()
    a = f32(host_bits(out_d[0])).reshape(2, 8, 128)[same]
    b = f32(host_bits(out_p[0, L])).reshape(2, 8, 128)[same]
    assert np.abs(a - b).max() <= 1.6e-2
    np.testing.assert_allclose(lse_d[0].cpu().numpy().reshape(2, 8)[same], lse_p[0, L].cpu().numpy().reshape(2, 8)[same],
                               rtol=0, atol=1e-3)


def test_appends_reproduce_block_pooling(cuda_ok):
    G, n = 2, 128 * 3
    k_idx = synth.normal_bf16(5, synth.STREAM_KI, (1, n, G, 64))
    shape = Shape.make(1, 8, G)
    ref = torch.zeros(1, G, 4, 64, device="cuda")
    msa_pool_index_keys(shape, dev_bf16(k_idx), n, ref, 4, None)
    pooled = torch.zeros(1, G, 4, 64, device="cuda")
    tail = torch.zeros(1, G, 64, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    kd = dev_bf16(k_idx)
    for pos in range(n):
        ctx = torch.tensor([pos], dtype=torch.int32, device="cuda")
        msa_pooled_keys_append(shape, kd[:, pos].contiguous(), None, None, ctx, None, None, 0, tail, pooled, 4, ws)
    torch.cuda.synchronize()
    assert msa_get_device_status(ws)[0] == 0
    np.testing.assert_allclose(pooled[:, :, :3].cpu().numpy(), ref[:, :, :3].cpu().numpy(), rtol=1e-5, atol=1e-6)


def test_device_bounds_are_reported_not_faulted(cuda_ok):
    shape = Shape.make(2, 8, 1)
    max_pos = 1000
    bufs = pipeline.decode_buffers(2, 8, 1, max_pos, "cuda")
    q_idx = torch.zeros(2, 1, 64, dtype=torch.bfloat16, device="cuda")
    pooled = torch.zeros(2, 1, 8, 64, device="cuda")
    q_pos = torch.tensor([5, 5000], dtype=torch.int32, device="cuda")   # second is beyond max_pos
    msa_index_select(shape, q_idx, 1, q_pos, max_pos, pooled, 8, bufs["sel"], bufs["ws_select"])
    st, info = msa_get_device_status(bufs["ws_select"])
    assert st == 6 and info[3] == 5000
    assert msa_get_device_status(bufs["ws_select"])[0] == 0          # cleared after reading


@pytest.mark.parametrize("case", ["many_survivors", "all_equal", "random"])
def test_decode_select_long_context_merge(cuda_ok, case):
    """Selection over 10,240 candidate blocks (80 chunks of 128 per query): the merge of the
    chunks' best-15 lists against the oracle, including lists built so that more than a
    thousand keys tie with or exceed the largest 15th key (the merge's slow path) and pooled
    keys that are all equal (ties to the lower id everywhere)."""
    c = 10240
    pos = c * 128 + 5
    nb_cap = c + 1
    q_bits = np.zeros((1, 1, 64), np.uint16)
    pooled = np.zeros((1, 1, nb_cap, 64), np.float32)
    if case == "random":
        q_bits = synth.normal_bf16(77, synth.STREAM_QI, (1, 1, 64))
        pooled[..., :] = synth.bf16_bits_to_f32(synth.normal_bf16(78, synth.STREAM_KI, (1, 1, nb_cap, 64)))
    else:
        q_bits[..., 0] = 0x3F80                       # q_I = e_0: the score of block j is pooled[j, 0] / 8
        if case == "many_survivors":
            # chunk 0: 15 blocks at 5; chunks 1..79: 14 blocks at 10 and the rest at 0, so every
            # list but the first has its 15th key at score 0 and ~1,100 keys survive the bound
            pooled[0, 0, :15, 0] = 5.0
            for ch in range(1, c // 128):
                pooled[0, 0, ch * 128:ch * 128 + 14, 0] = 10.0
        else:
            pooled[..., 0] = 1.0
    shape = Shape.make(1, 4, 1)
    bufs = pipeline.decode_buffers(1, 4, 1, pos, "cuda")
    q_pos = torch.tensor([pos], dtype=torch.int32, device="cuda")
    msa_index_select(shape, dev_bf16(q_bits), 1, q_pos, pos, torch.from_numpy(pooled).cuda(), nb_cap,
                     bufs["sel"], bufs["ws_select"])
    torch.cuda.synchronize()
    assert msa_get_device_status(bufs["ws_select"])[0] == 0
    sel = bufs["sel"].cpu().numpy()[0, 0]
    ref, kth, _ = oracle.select_rows(np.array([pos]), q_bits[0], pooled[0, 0].astype(np.float64))
    check_selection(sel[None], ref, kth, q_bits[0], pooled[0, 0].astype(np.float64), np.array([pos]),
                    label=f"decode 10,240 candidates ({case})")
    if case != "random":
        assert (sel == ref[0]).all(), (case, sel, ref[0])
    if case == "many_survivors":
        assert list(sel) == list(range(128, 142)) + [256, c]


@pytest.mark.parametrize("order", ["append-select-attend", "select-append-attend"])
def test_decode_step_order_gives_the_same_results(cuda_ok, order):
    """The append may run before or after the step's selection (the selection scores only blocks
    below the new token's own, and the append runs under programmatic dependent launch in the
    shadow of the kernel before it): both orders, eager and replayed from a graph, give the
    pipeline's selection exactly and its output and lse up to the order of the fp32 merge of a
    group split over CTAs (whichever CTA arrives last merges), and a block that the step closes
    is pooled."""
    w = synth.Workload(name="t", kind="decode", B=3, Hq=16, G=2, ctx=(2047, 3000, 383), seed=4242)
    l_cap = 3200
    ref = build_decode_state(w, l_cap)
    o_ref, l_ref, s_ref = run_step(w, ref)
    for graph in (False, True):
        st = build_decode_state(w, l_cap)
        s, mp = Shape.make(w.B, w.Hq, w.G), max(w.ctx)
        bufs = pipeline.decode_buffers(w.B, w.Hq, w.G, mp, "cuda")

        def step():
            app = lambda: msa_pooled_keys_append(s, st["k_idx_new"], st["k_new"], st["v_new"], st["ctx"],  # noqa: E731
                                                 st["k_cache"], st["v_cache"], l_cap, st["tail"], st["pooled"],
                                                 st["nb_cap"], bufs["ws_append"])
            sel = lambda: msa_index_select(s, st["q_idx"], 1, st["ctx"], mp, st["pooled"], st["nb_cap"],  # noqa: E731
                                           bufs["sel"], bufs["ws_select"])
            for f in ((app, sel) if order == "append-select-attend" else (sel, app)):
                f()
            msa_sparse_attn_decode(s, st["q"], st["k_cache"], st["v_cache"], l_cap, st["ctx"], mp, bufs["sel"],
                                   bufs["out"], bufs["lse"], bufs["ws_attn"])

        if graph:
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step()
            g.replay()
        else:
            step()
        torch.cuda.synchronize()
        for key in ("ws_append", "ws_select", "ws_attn"):
            stt, info = msa_get_device_status(bufs[key])
            assert stt == 0, (key, stt, info)
        assert np.array_equal(bufs["sel"].cpu().numpy(), s_ref)
        o = f32(host_bits(bufs["out"]))
        assert (np.abs(o - o_ref) <= np.abs(o_ref) * 2.0 ** -7 + 1e-6).all()    # one bf16 step at most
        np.testing.assert_allclose(bufs["lse"].cpu().numpy(), l_ref, rtol=1e-6, atol=1e-6)
        # sequence 0 (2,047 cached tokens) closes block 15 with this step
        assert torch.equal(st["pooled"][0, :, 15], ref["pooled"][0, :, 15])
        assert not torch.isnan(st["pooled"][0, :, 15]).any()
        if graph:
            del g


def test_decode_step_entry_matches_separate_calls(cuda_ok):
    """msa_decode_step (80 groups: one attention CTA per (sequence, group)) gives the selection,
    output and lse of the three separate calls bit for bit, eager and replayed from a graph, call
    after call, writes the same cache rows, and leaves no device error."""
    w = synth.Workload(name="t", kind="decode", B=10, Hq=64, G=8,
                       ctx=(2047, 3000, 383, 4095, 128, 2500, 1000, 3333, 127, 3900), seed=777)
    l_cap = 4224
    s, mp = Shape.make(w.B, w.Hq, w.G), max(w.ctx)
    ref = build_decode_state(w, l_cap)
    rb = pipeline.decode_buffers(w.B, w.Hq, w.G, mp, "cuda")
    msa_index_select(s, ref["q_idx"], 1, ref["ctx"], mp, ref["pooled"], ref["nb_cap"], rb["sel"], rb["ws_select"])
    msa_pooled_keys_append(s, ref["k_idx_new"], ref["k_new"], ref["v_new"], ref["ctx"], ref["k_cache"],
                           ref["v_cache"], l_cap, ref["tail"], ref["pooled"], ref["nb_cap"], rb["ws_append"])
    msa_sparse_attn_decode(s, ref["q"], ref["k_cache"], ref["v_cache"], l_cap, ref["ctx"], mp, rb["sel"], rb["out"],
                           rb["lse"], rb["ws_attn"])
    torch.cuda.synchronize()
    s_ref, o_ref, l_ref = rb["sel"].clone(), rb["out"].clone(), rb["lse"].clone()

    st = build_decode_state(w, l_cap)
    bufs = pipeline.decode_buffers(w.B, w.Hq, w.G, mp, "cuda")

    def step():
        pipeline.decode_step(st["q"], st["q_idx"], st["k_idx_new"], st["k_new"], st["v_new"], st["ctx"],
                             st["k_cache"], st["v_cache"], st["tail"], st["pooled"], bufs)

    def check(what):
        torch.cuda.synchronize()
        for key in ("ws_append", "ws_select", "ws_attn"):
            stt, info = msa_get_device_status(bufs[key])
            assert stt == 0, (what, key, stt, info)
        assert torch.equal(bufs["sel"], s_ref), what
        assert torch.equal(bufs["out"].view(torch.int16), o_ref.view(torch.int16)), what
        assert torch.equal(bufs["lse"], l_ref), what
        bufs["out"].zero_()
        bufs["sel"].fill_(-7)

    for i in range(3):
        step()
        check(f"eager call {i}")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for i in range(3):
        g.replay()
        check(f"graph replay {i}")
    del g
    for key in ("k_cache", "v_cache"):          # bits: rows past the context hold NaNs
        assert torch.equal(st[key].view(torch.int16), ref[key].view(torch.int16)), key
