"""GPU parity of the main branch's backward pass (dQ, dK, dV over the selected keys, the
selection held fixed) against the fp64 oracle of the gradient, through the C ABI, on the GPU's
own forward selection. Sources: youmind article "MiniMax M3 sparse attention agents", bullet on
MSA-CPT; KuCoin flash "MiniMax launches MSA sparse attention method and MiniMax-M3 model",
"ME AI News" (MSA-PT). Tolerance: tests/msa_check.py (relative to the gradient's magnitude,
from the bf16 roundings of p and dS)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from block_sparse_gqa_branch_b200 import msa_get_device_status, pipeline
from tests.gpu_util import dev_bf16
from tests.msa_check import assert_close_gradient

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,Hq,G", [(2304 + 37, 4, 1), (2600, 8, 2), (1500, 16, 1), (3000, 2, 2)])
def test_backward_matches_oracle(cuda_ok, N, Hq, G):
    w = synth.Workload(name="bwd", kind="prefill", B=1, N=N, Hq=Hq, G=G, seed=7000 + N)
    x = synth.prefill_inputs_np(w)
    d_out_bits = synth.normal_bf16(w.seed + 99, synth.STREAM_Q, (1, N, Hq, 128))
    d = {k: dev_bf16(v) for k, v in x.items()}
    fwd = pipeline.prefill_buffers(1, N, Hq, G, "cuda")
    pipeline.prefill(d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], fwd)
    bwd = pipeline.backward_buffers(1, N, Hq, G, "cuda")
    dq, dk, dv = pipeline.prefill_backward(d["q"], d["k"], d["v"], dev_bf16(d_out_bits), fwd, bwd)
    torch.cuda.synchronize()
    for key, buf in (("ws_attn", fwd["ws_attn"]), ("ws_bwd", bwd["ws"])):
        st, info = msa_get_device_status(buf)
        assert st == 0, (key, st, info)
    sel = fwd["sel"][0].cpu().numpy()
    dq, dk, dv = dq[0].cpu().numpy(), dk[0].cpu().numpy(), dv[0].cpu().numpy()
    Hg = Hq // G
    t = np.arange(N)
    dO = synth.bf16_bits_to_f32(d_out_bits[0]).astype(np.float64)
    for g in range(G):
        rq, rk, rv = oracle.attend_grad(t, x["q"][0, :, g * Hg:(g + 1) * Hg], x["k"][0, g], x["v"][0, g], sel[:, g],
                                        dO[:, g * Hg:(g + 1) * Hg])
        assert_close_gradient(dq[:, g * Hg:(g + 1) * Hg], rq, f"dQ N={N} g={g}")
        assert_close_gradient(dk[g], rk, f"dK N={N} g={g}")
        assert_close_gradient(dv[g], rv, f"dV N={N} g={g}")
