"""GPU parity of chunked prefill (a chunk of queries at positions P .. P + n - 1 against caches
that hold the earlier positions) against the fp64 oracle, through the C ABI. Source: youmind
article "MiniMax M3 sparse attention agents", bullet "Predictable cost at every length" (the
same 16-block budget at every length).

A sequence is prefilled in chunks of ragged sizes (chunk starts inside blocks, a one-token
chunk, a chunk inside one block); after every chunk: pooled keys and the running sum of the
open block against the oracle, selection exact outside logged near-ties, attention on the GPU's
own selection within max |err| <= 2e-2, mean |err| <= 2e-3, lse within 2e-3. Cache rows past
the chunk hold NaN, which must never reach an output. Where the chunked selection equals the
whole prefill's, the chunked output must equal the whole prefill's rows bit for bit (each
partial row and the merge depend only on the query and its selection)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from block_sparse_gqa_branch_b200 import msa_get_device_status, pipeline
from tests.gpu_util import check_selection, dev_bf16, f32, host_bits
from tests.msa_check import assert_close_attention

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC0


@pytest.mark.parametrize("N,Hq,G,chunks", [
    (3100, 16, 2, [700, 1100, 1, 60, 1239]),
    (4000, 64, 8, [2500, 1500]),
    (2300, 8, 1, [128, 2047, 125]),
    # the last chunk scores up to 78 candidates: two 64-candidate chunks of split pooled keys
    (10050, 16, 2, [8100, 1950]),
])
def test_chunked_prefill_matches_oracle(cuda_ok, N, Hq, G, chunks):
    assert sum(chunks) == N
    w = synth.Workload(name="chunk", kind="prefill", B=1, N=N, Hq=Hq, G=G, seed=555 + N)
    x = synth.prefill_inputs_np(w)
    d = {k: dev_bf16(v) for k, v in x.items()}
    l_cap = (N + 127) // 128 * 128 + 256
    k_cache = torch.empty(1, G, l_cap, 128, dtype=torch.bfloat16, device="cuda")
    v_cache = torch.empty_like(k_cache)
    k_cache.view(torch.int16).fill_(NAN_BF16)
    v_cache.view(torch.int16).fill_(NAN_BF16)
    nb_cap = l_cap // 128
    pooled = torch.full((1, G, nb_cap, 64), float("nan"), device="cuda")
    tail = torch.zeros(1, G, 64, device="cuda")
    # the whole prefill, for the bit-for-bit comparison
    wbufs = pipeline.prefill_buffers(1, N, Hq, G, "cuda")
    w_out, w_lse, w_sel = pipeline.prefill(d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], wbufs)
    torch.cuda.synchronize()
    w_out, w_sel = host_bits(w_out)[0], w_sel[0].cpu().numpy()
    P = 0
    same_rows = 0
    for n in chunks:
        # the chunk's K and V rows go into the caches; positions past P + n stay NaN
        k_cache[:, :, P:P + n] = d["k"][:, :, P:P + n]
        v_cache[:, :, P:P + n] = d["v"][:, :, P:P + n]
        out, lse, sel, ws = pipeline.prefill_chunk(d["q"][:, P:P + n].contiguous(), d["q_idx"][:, P:P + n].contiguous(),
                                                   d["k_idx"][:, P:P + n].contiguous(), k_cache, v_cache, P, pooled,
                                                   tail, Hq)
        torch.cuda.synchronize()
        for key in ("ws_select", "ws_attn"):
            st, info = msa_get_device_status(ws[key])
            assert st == 0, (key, st, info)
        ref = oracle.prefill_chunk(x["q"][0, P:P + n], x["q_idx"][0, P:P + n], x["k_idx"][0], x["k"][0], x["v"][0],
                                   P, Hq, G, sel=sel[0].cpu().numpy())
        nb = (P + n) // 128
        np.testing.assert_allclose(pooled[0, :, :nb].cpu().numpy(), ref["pooled"][:, :nb], rtol=1e-6, atol=1e-7)
        _, rtail = oracle.pool(x["k_idx"][0, :P + n], 128)
        np.testing.assert_allclose(tail[0].cpu().numpy(), rtail, rtol=1e-5, atol=1e-5)
        sel_h = sel[0].cpu().numpy()
        t = np.arange(P, P + n)
        for g in range(G):
            check_selection(sel_h[:, g], ref["sel"][:, g], ref["kth"][:, g], x["q_idx"][0, P:P + n, g],
                            ref["pooled"][g], t, label=f"chunked prefill N={N} chunks={chunks}")
        got = f32(host_bits(out[0]))
        assert_close_attention(got, ref["out"], f"chunk P={P} n={n}")
        np.testing.assert_allclose(lse[0].cpu().numpy(), ref["lse"], rtol=0, atol=2e-3)
        eq = (sel_h == w_sel[P:P + n]).all(axis=(1, 2))
        same_rows += int(eq.sum())
        assert (host_bits(out[0])[eq] == w_out[P:P + n][eq]).all(), f"chunk P={P}: rows differ from the whole prefill"
        P += n
    assert same_rows > N // 2
