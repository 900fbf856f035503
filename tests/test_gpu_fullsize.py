"""Parity at the full sizes of the five benchmark workloads, in the launch configuration the
bench times (same entry points, shapes and buffers). The GPU runs the whole problem; the
oracle recomputes from inputs regenerated on the host with the same counter-based generator:

* prefill 32K (planted) and 128K: the block selection of EVERY (token, group) row (exact
  outside logged near-ties), and attention on the GPU's own selection (max |err| <= 2e-2,
  mean |err| <= 2e-3, lse within 2e-3) for 1,024 random tokens of every group plus the first
  and last 128 tokens of every group (8,192 random rows in all, plus 2,048 edge rows);
* prefill 4K: every row of selection and attention;
* decode batch 16 at 128K and the ragged 1M batch: every (sequence, group) pair.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth
from block_sparse_gqa_branch_b200 import msa_get_device_status, pipeline
from tests.gpu_util import check_selection, f32, host_bits
from tests.msa_check import assert_close_attention

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _attention_tokens(N, n_random, seed):
    """n_random uniform tokens plus the first and last 128 tokens (and the budget edges)."""
    rng = np.random.default_rng(seed)
    edge = list(range(min(128, N))) + list(range(max(0, N - 128), N)) + [2047, 2048, 2049, N // 2]
    t = np.concatenate([np.array([e for e in edge if 0 <= e < N]), rng.integers(0, N, n_random)])
    return np.unique(t)


def _prefill_host_rows(w, g, t):
    """Host bits for the oracle: q rows [n, Hg, d] of group g at tokens t, and the group's K, V."""
    Hg = w.Hq // w.G
    h = np.arange(g * Hg, (g + 1) * Hg, dtype=np.uint64)
    e = np.arange(w.d, dtype=np.uint64)
    idx = ((t.astype(np.uint64)[:, None, None] * np.uint64(w.Hq) + h[None, :, None]) * np.uint64(w.d)
           + e[None, None, :])
    q = synth.normal_bf16_at(w.seed, synth.STREAM_Q, idx)
    start = g * w.N * w.d                                    # batch 1: k, v are [1, G, N, d]
    K = synth.normal_bf16(w.seed, synth.STREAM_K, (w.N, w.d), start=start)
    V = synth.normal_bf16(w.seed, synth.STREAM_V, (w.N, w.d), start=start)
    return q, K, V


def _check_prefill(wname, n_random_per_group, seed):
    w = synth.WORKLOADS[wname]
    assert w.B == 1
    x = synth.prefill_inputs_torch(w, "cuda")
    bufs = pipeline.prefill_buffers(w.B, w.N, w.Hq, w.G, "cuda")
    out, lse, sel = pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], bufs)
    torch.cuda.synchronize()
    assert msa_get_device_status(bufs["ws_select"])[0] == 0
    assert msa_get_device_status(bufs["ws_attn"])[0] == 0
    del x
    sel_h = sel[0].cpu().numpy()                             # [N, G, 16]
    # oracle inputs: every index key and index query (selection is checked on every row),
    # planted as on the GPU
    k_idx = synth.normal_bf16(w.seed, synth.STREAM_KI, (w.B, w.N, w.G, w.dI))
    q_idx = synth.normal_bf16(w.seed, synth.STREAM_QI, (w.B, w.N, w.G, w.dI))
    if w.planted:
        shift, blocks = synth.plant_plan(w, q_idx)
        k_idx = synth.apply_plant_np(k_idx, shift, blocks, w.Bk)
    pooled, _ = oracle.pool(k_idx[0], w.Bk)
    del k_idx
    t_all = np.arange(w.N)
    Hg = w.Hq // w.G
    for g in range(w.G):
        ref, kth, _ = oracle.select_rows(t_all, q_idx[0, :, g], pooled[g])
        check_selection(sel_h[:, g], ref, kth, q_idx[0, :, g], pooled[g], t_all, label=f"{wname} (every row)")
        t = _attention_tokens(w.N, n_random_per_group, seed + g)
        tt = torch.from_numpy(t).cuda()
        qr, K, V = _prefill_host_rows(w, g, t)
        o, l, _ = oracle.attend_rows(t, qr, K, V, sel_h[t, g])
        got = f32(host_bits(out[0, tt, g * Hg:(g + 1) * Hg]))
        assert_close_attention(got, o, f"{wname} g={g}")
        np.testing.assert_allclose(lse[0, tt, g * Hg:(g + 1) * Hg].cpu().numpy(), l, rtol=0, atol=2e-3)


def test_prefill_4k_h4g1_every_row(cuda_ok):
    w = synth.WORKLOADS["prefill_4k_h4g1"]
    x = synth.prefill_inputs_np(w)
    d = {k: torch.from_numpy(v.view(np.int16)).cuda().view(torch.bfloat16) for k, v in x.items()}
    bufs = pipeline.prefill_buffers(w.B, w.N, w.Hq, w.G, "cuda")
    out, lse, sel = pipeline.prefill(d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], bufs)
    torch.cuda.synchronize()
    pooled, _ = oracle.pool(x["k_idx"][0], w.Bk)
    t = np.arange(w.N)
    ref, kth, _ = oracle.select_rows(t, x["q_idx"][0, :, 0], pooled[0])
    gsel = sel[0, :, 0].cpu().numpy()
    check_selection(gsel, ref, kth, x["q_idx"][0, :, 0], pooled[0], t, label="prefill_4k_h4g1 (every row)")
    o, l, _ = oracle.attend_rows(t, x["q"][0], x["k"][0, 0], x["v"][0, 0], gsel)
    assert_close_attention(f32(host_bits(out[0])), o, "prefill_4k_h4g1")
    np.testing.assert_allclose(lse[0].cpu().numpy(), l, rtol=0, atol=2e-3)


def test_prefill_32k_planted_every_selection_row(cuda_ok):
    _check_prefill("prefill_32k_h64g8_planted", 1024, seed=11)


def test_prefill_128k_every_selection_row(cuda_ok):
    _check_prefill("prefill_128k_h64g8", 1024, seed=12)


def _check_decode(wname):
    w = synth.WORKLOADS[wname]
    ds = bench.build_decode_state(w, torch.device("cuda"))
    bufs = pipeline.decode_buffers(w.B, w.Hq, w.G, max(w.ctx), "cuda")
    out, lse, sel = pipeline.decode_step(ds["q"], ds["q_idx"], ds["k_idx_new"], ds["k_new"], ds["v_new"], ds["ctx"],
                                         ds["k_cache"], ds["v_cache"], ds["tail"], ds["pooled"], bufs)
    torch.cuda.synchronize()
    for k in ("ws_append", "ws_select", "ws_attn"):
        assert msa_get_device_status(bufs[k])[0] == 0, k
    out, lse, sel = f32(host_bits(out)), lse.cpu().numpy(), sel.cpu().numpy()
    del ds
    Hg = w.Hq // w.G
    for b in range(w.B):
        Lb = w.ctx[b]                                       # the new token's position
        t = np.array([Lb])
        ki = synth.decode_seq_np(w, b, "k_idx")             # [Lb + 1, G, dI]
        pooled, _ = oracle.pool(ki, w.Bk)
        del ki
        qi_all = synth.decode_seq_np(w, b, "q_idx")
        q_all = synth.decode_seq_np(w, b, "q")
        for g in range(w.G):
            qi = qi_all[g][None]
            ref, kth, _ = oracle.select_rows(t, qi, pooled[g])
            check_selection(sel[b, g][None], ref, kth, qi, pooled[g], t, label=f"{wname} (every pair)")
            # K, V: only the selected blocks' rows are read by the oracle
            K = np.zeros((Lb + 1, w.d), np.uint16)
            V = np.zeros((Lb + 1, w.d), np.uint16)
            for j in sel[b, g]:
                if j < 0:
                    continue
                lo, hi = j * w.Bk, min((j + 1) * w.Bk, Lb + 1)
                K[lo:hi] = synth.decode_seq_np(w, b, "k", lo, hi, g=g)
                V[lo:hi] = synth.decode_seq_np(w, b, "v", lo, hi, g=g)
            q = q_all[g * Hg:(g + 1) * Hg][None]
            o, l, _ = oracle.attend_rows(t, q, K, V, sel[b, g][None])
            assert_close_attention(out[b, g * Hg:(g + 1) * Hg][None], o, f"{wname} b={b} g={g}")
            np.testing.assert_allclose(lse[b, g * Hg:(g + 1) * Hg], l[0], rtol=0, atol=2e-3)


def test_decode_128k_b16_every_pair(cuda_ok):
    _check_decode("decode_128k_b16_h64g8")


def test_decode_1m_ragged_every_pair(cuda_ok):
    _check_decode("decode_1m_ragged_b4_h64g8")
