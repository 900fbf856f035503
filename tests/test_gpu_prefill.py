"""GPU parity of the prefill path (pooling, selection, main branch) against the fp64 oracle,
through the C ABI, on seeded inputs spanning several blocks and ragged tails."""
import numpy as np
import pytest
import torch

import oracle
import synth
from block_sparse_gqa_branch_b200 import Shape, msa_get_device_status, msa_pool_index_keys, pipeline
from tests.gpu_util import check_selection, dev_bf16, f32, host_bits
from tests.msa_check import assert_close_attention

pytestmark = pytest.mark.gpu


def run_prefill(w, x):
    d = {k: dev_bf16(v) for k, v in x.items()}
    bufs = pipeline.prefill_buffers(w.B, w.N, w.Hq, w.G, "cuda")
    out, lse, sel = pipeline.prefill(d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], bufs)
    torch.cuda.synchronize()
    for key in ("ws_select", "ws_attn"):
        st, info = msa_get_device_status(bufs[key])
        assert st == 0, (key, st, info)
    return {"out": f32(host_bits(out)), "lse": lse.cpu().numpy(), "sel": sel.cpu().numpy(),
            "pooled": bufs["pooled"].cpu().numpy(), "tail": bufs["tail_sum"].cpu().numpy()}


@pytest.mark.parametrize("N,G", [(1000, 2), (4096, 1), (131, 3)])
def test_pool_matches_oracle(cuda_ok, N, G):
    w = synth.small_workload(N=N, Hq=G, G=G, B=2, seed=N + G)
    k_idx = synth.normal_bf16(w.seed, synth.STREAM_KI, (2, N, G, 64))
    shape = Shape.make(2, G, G)
    nb = N // 128
    pooled = torch.full((2, G, max(nb, 1), 64), 7.0, device="cuda")
    tail = torch.full((2, G, 64), 7.0, device="cuda")
    msa_pool_index_keys(shape, dev_bf16(k_idx), N, pooled, max(nb, 1), tail)
    torch.cuda.synchronize()
    for b in range(2):
        ref, rtail = oracle.pool(k_idx[b], 128)
        got = pooled[b, :, :nb].cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-7)
        np.testing.assert_allclose(tail[b].cpu().numpy(), rtail, rtol=1e-6, atol=1e-5)


@pytest.mark.parametrize("N,Hq,G,planted", [(4096, 4, 1, 0), (2500, 8, 2, 0), (128 * 40 + 77, 16, 2, 8),
                                            (3000, 16, 1, 0), (2177, 2, 2, 0), (640, 4, 4, 0), (1500, 4, 2, 0)])
def test_prefill_matches_oracle(cuda_ok, N, Hq, G, planted):
    w = synth.Workload(name="t", kind="prefill", B=1, N=N, Hq=Hq, G=G, seed=1000 + N, planted=planted)
    x = synth.prefill_inputs_np(w)
    r = run_prefill(w, x)
    o = oracle.prefill(x, Hq, G, sel=r["sel"])
    # selection: exact except logged near-ties
    t = np.arange(N)
    for g in range(G):
        check_selection(r["sel"][0, :, g], o["sel"][0, :, g], o["kth"][0, :, g], x["q_idx"][0, :, g],
                        o["pooled"][0, g], t, label=f"prefill N={N} Hq={Hq} G={G} planted={planted}")
    # pooled keys
    nb = N // 128
    np.testing.assert_allclose(r["pooled"][0, :, :nb], o["pooled"][0], rtol=1e-6, atol=1e-7)
    # attention on the GPU's own selection
    assert_close_attention(r["out"], o["out"], f"prefill N={N} Hq={Hq} G={G}")
    np.testing.assert_allclose(r["lse"], o["lse"], rtol=0, atol=2e-3)


def test_prefill_equal_scores_take_lowest_blocks(cuda_ok):
    # constant index keys: every score ties -> {0..14, c} for every query with c >= 15
    w = synth.Workload(name="t", kind="prefill", B=1, N=128 * 20 + 5, Hq=8, G=1, seed=77)
    x = synth.prefill_inputs_np(w)
    x["k_idx"][:] = synth.f64_to_bf16_bits(np.array([0.5]))[0]
    r = run_prefill(w, x)
    for t in [2048, 2049, 128 * 20, 128 * 20 + 4]:
        c = t // 128
        assert list(r["sel"][0, t, 0]) == list(range(15)) + [c]
    x2 = synth.prefill_inputs_np(w)
    x2["q_idx"][:] = 0
    r2 = run_prefill(w, x2)
    assert list(r2["sel"][0, 2560, 0]) == list(range(15)) + [20]


def test_prefill_constant_v_gives_v(cuda_ok):
    w = synth.Workload(name="t", kind="prefill", B=1, N=2304 + 50, Hq=8, G=1, seed=78)
    x = synth.prefill_inputs_np(w)
    x["v"][:] = synth.f64_to_bf16_bits(np.array([0.625]))[0]
    r = run_prefill(w, x)
    assert np.abs(r["out"] - 0.625).max() == 0.0


def test_prefill_batch_of_two(cuda_ok):
    w = synth.Workload(name="t", kind="prefill", B=2, N=2400, Hq=8, G=2, seed=79)
    x = synth.prefill_inputs_np(w)
    r = run_prefill(w, x)
    o = oracle.prefill(x, 8, 2, sel=r["sel"])
    for b in range(2):
        for g in range(2):
            check_selection(r["sel"][b, :, g], o["sel"][b, :, g], o["kth"][b, :, g], x["q_idx"][b, :, g],
                            o["pooled"][b, g], np.arange(2400), label="prefill batch 2 N=2400")
    assert_close_attention(r["out"], o["out"], "batch 2")


@pytest.mark.parametrize("B,N,Hq,G", [(2, 2100, 16, 8), (1, 16384 + 700, 8, 8)])
def test_prefill_many_groups_and_two_ranges(cuda_ok, B, N, Hq, G):
    """Eight groups over two sequences, and a sequence whose queries span two 16K-token ranges of
    the inverted index (the second one ragged). Same bar as the other prefill cases, and the
    outputs equal a second call bit for bit."""
    w = synth.Workload(name="t", kind="prefill", B=B, N=N, Hq=Hq, G=G, seed=N + B)
    x = synth.prefill_inputs_np(w)
    r = run_prefill(w, x)
    r2 = run_prefill(w, x)
    assert np.array_equal(r["out"], r2["out"]) and np.array_equal(r["lse"], r2["lse"])
    o = oracle.prefill(x, Hq, G, sel=r["sel"])
    for b in range(B):
        for g in range(G):
            check_selection(r["sel"][b, :, g], o["sel"][b, :, g], o["kth"][b, :, g], x["q_idx"][b, :, g],
                            o["pooled"][b, g], np.arange(N), label=f"prefill B={B} N={N} G={G}")
    assert_close_attention(r["out"], o["out"], f"prefill B={B} N={N} G={G}")
    np.testing.assert_allclose(r["lse"], o["lse"], rtol=0, atol=2e-3)
