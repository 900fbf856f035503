"""Parity at the full sizes of the five benchmark workloads, in the launch configuration the
bench times (same entry points, shapes and buffers). The GPU runs the whole problem; the
oracle recomputes sampled rows one by one from inputs regenerated on the host with the same
counter-based generator: block selection (exact outside logged near-ties) and attention on
the GPU's own selection (max |err| <= 2e-2, mean |err| <= 2e-3, lse within 2e-3)."""
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


def _sample_tokens(N, n, seed):
    rng = np.random.default_rng(seed)
    edge = [0, 1, 127, 128, 129, 2047, 2048, 2049, N // 2, N - 129, N - 128, N - 2, N - 1]
    t = np.concatenate([np.array([e for e in edge if 0 <= e < N]), rng.integers(0, N, n)])
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


def _check_prefill(wname, n_samples, groups, seed):
    w = synth.WORKLOADS[wname]
    assert w.B == 1
    x = synth.prefill_inputs_torch(w, "cuda")
    bufs = pipeline.prefill_buffers(w.B, w.N, w.Hq, w.G, "cuda")
    out, lse, sel = pipeline.prefill(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], bufs)
    torch.cuda.synchronize()
    assert msa_get_device_status(bufs["ws_attn"])[0] == 0
    del x
    # oracle inputs: the whole index keys (pooling needs every block), planted as on the GPU;
    # the index queries of the sampled tokens (all of them when planting needs their mean)
    t = _sample_tokens(w.N, n_samples, seed)
    k_idx = synth.normal_bf16(w.seed, synth.STREAM_KI, (w.B, w.N, w.G, w.dI))
    if w.planted:
        q_idx_all = synth.normal_bf16(w.seed, synth.STREAM_QI, (w.B, w.N, w.G, w.dI))
        shift, blocks = synth.plant_plan(w, q_idx_all)
        k_idx = synth.apply_plant_np(k_idx, shift, blocks, w.Bk)
        q_idx = q_idx_all[0, t]                              # [n, G, dI]
    else:
        gg = np.arange(w.G, dtype=np.uint64)
        e = np.arange(w.dI, dtype=np.uint64)
        idx = (t.astype(np.uint64)[:, None, None] * np.uint64(w.G) + gg[None, :, None]) * np.uint64(w.dI) + e
        q_idx = synth.normal_bf16_at(w.seed, synth.STREAM_QI, idx)
    pooled, _ = oracle.pool(k_idx[0], w.Bk)
    del k_idx
    tt = torch.from_numpy(t).cuda()
    Hg = w.Hq // w.G
    for g in groups:
        gsel = sel[0, tt, g].cpu().numpy()
        ref, kth, _ = oracle.select_rows(t, q_idx[:, g], pooled[g])
        check_selection(gsel, ref, kth, q_idx[:, g], pooled[g], t)
        qr, K, V = _prefill_host_rows(w, g, t)
        o, l, _ = oracle.attend_rows(t, qr, K, V, gsel)
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
    check_selection(gsel, ref, kth, x["q_idx"][0, :, 0], pooled[0], t)
    o, l, _ = oracle.attend_rows(t, x["q"][0], x["k"][0, 0], x["v"][0, 0], gsel)
    assert_close_attention(f32(host_bits(out[0])), o, "prefill_4k_h4g1")
    np.testing.assert_allclose(lse[0].cpu().numpy(), l, rtol=0, atol=2e-3)


def test_prefill_32k_planted_sampled(cuda_ok):
    _check_prefill("prefill_32k_h64g8_planted", 48, range(8), seed=11)


def test_prefill_128k_sampled(cuda_ok):
    _check_prefill("prefill_128k_h64g8", 40, (0, 5), seed=12)


def _check_decode(wname, pairs):
    w = synth.WORKLOADS[wname]
    ds = bench.build_decode_state(w, torch.device("cuda"))
    bufs = pipeline.decode_buffers(w.B, w.Hq, w.G, max(w.ctx), "cuda")
    out, lse, sel = pipeline.decode_step(ds["q"], ds["q_idx"], ds["k_idx_new"], ds["k_new"], ds["v_new"], ds["ctx"],
                                         ds["k_cache"], ds["v_cache"], ds["tail"], ds["pooled"], bufs)
    torch.cuda.synchronize()
    for k in ("ws_append", "ws_select", "ws_attn"):
        assert msa_get_device_status(bufs[k])[0] == 0, k
    out, lse, sel = f32(host_bits(out)), lse.cpu().numpy(), sel.cpu().numpy()
    Hg = w.Hq // w.G
    for b, g in pairs:
        Lb = w.ctx[b]                                       # the new token's position
        t = np.array([Lb])
        ki = synth.decode_seq_np(w, b, "k_idx", g=g)        # [Lb + 1, dI]
        pooled, _ = oracle.pool(ki[:, None, :], w.Bk)
        qi = synth.decode_seq_np(w, b, "q_idx")[g][None]
        ref, kth, _ = oracle.select_rows(t, qi, pooled[0])
        check_selection(sel[b, g][None], ref, kth, qi, pooled[0], t)
        # K, V: only the selected blocks' rows are read by the oracle
        K = np.zeros((Lb + 1, w.d), np.uint16)
        V = np.zeros((Lb + 1, w.d), np.uint16)
        for j in sel[b, g]:
            if j < 0:
                continue
            lo, hi = j * w.Bk, min((j + 1) * w.Bk, Lb + 1)
            K[lo:hi] = synth.decode_seq_np(w, b, "k", lo, hi, g=g)
            V[lo:hi] = synth.decode_seq_np(w, b, "v", lo, hi, g=g)
        q = synth.decode_seq_np(w, b, "q")[g * Hg:(g + 1) * Hg][None]
        o, l, _ = oracle.attend_rows(t, q, K, V, sel[b, g][None])
        assert_close_attention(out[b, g * Hg:(g + 1) * Hg][None], o, f"{wname} b={b} g={g}")
        np.testing.assert_allclose(lse[b, g * Hg:(g + 1) * Hg], l[0], rtol=0, atol=2e-3)


def test_decode_128k_b16_sampled(cuda_ok):
    _check_decode("decode_128k_b16_h64g8", [(0, 0), (3, 7), (7, 2), (9, 5), (12, 1), (15, 6)])


def test_decode_1m_ragged_sampled(cuda_ok):
    _check_decode("decode_1m_ragged_b4_h64g8", [(0, 3), (1, 0), (2, 7), (3, 4)])
