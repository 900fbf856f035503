"""GPU parity of the FP8 (e4m3) key-value cache decode variant against the fp64 oracle, through
the C ABI: the per-block quantisation (codes and scales bit for bit: both sides decide the code
in fp32), the block closed by a decode step's append, and the decode attention over the FP8
cache (closed blocks from codes x scale, the query's own block from bf16) on the GPU's own
selection within max |err| <= 2e-2, mean |err| <= 2e-3, lse within 2e-3.

Source: KuCoin flash "MiniMax launches MSA sparse attention method and MiniMax-M3 model", "ME AI
News" paragraph (the SM100 attention kernel also takes FP8 inputs)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from block_sparse_gqa_branch_b200 import Shape, msa_fp8_quantize_blocks, msa_get_device_status, pipeline
from tests.gpu_util import check_selection, f32, host_bits
from tests.msa_check import assert_close_attention
from tests.test_gpu_decode import build_decode_state

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("B,G,nblk", [(2, 2, 5), (1, 8, 3)])
def test_fp8_quantisation_matches_oracle_bit_for_bit(cuda_ok, B, G, nblk):
    l_cap = 128 * nblk + 64
    gen = torch.Generator(device="cuda").manual_seed(B * 100 + G)
    k = (torch.randn(B, G, l_cap, 128, device="cuda", generator=gen) * 1.7).to(torch.bfloat16)
    v = (torch.randn(B, G, l_cap, 128, device="cuda", generator=gen) * 0.3).to(torch.bfloat16)
    k[0, 0, 128:256] = 0                              # an all-zero block: scale 1, codes 0
    v[0, G - 1, 0, 5] = 3.0e4                         # one large value: the rest of its block goes subnormal
    k[B - 1, G - 1, 256 + 7, 100] = -2.0e-30          # tiny values round to (signed) zero codes
    f8 = pipeline.fp8_cache(k, v, nblk + 1)
    n_tokens = 128 * nblk + 50                        # the trailing partial block is not quantised
    msa_fp8_quantize_blocks(Shape.make(B, 8 * G, G), k, v, l_cap, n_tokens, f8["k_codes"], f8["v_codes"],
                            f8["k_scale"], f8["v_scale"], f8["nb_cap"])
    torch.cuda.synchronize()
    for b in range(B):
        for g in range(G):
            for name, src in (("k", k), ("v", v)):
                codes, scales = oracle.fp8_quantize_blocks(_bits(src[b, g, :128 * nblk]), 128)
                got_c = f8[name + "_codes"][b, g, :128 * nblk].cpu().numpy()
                got_s = f8[name + "_scale"][b, g, :nblk].cpu().numpy()
                assert (got_s.view(np.uint32) == scales.view(np.uint32)).all(), (name, b, g)
                assert (got_c == codes).all(), (name, b, g, np.argwhere(got_c != codes)[:5])
            # the block past n_tokens is left untouched
            assert float(f8["k_scale"][b, g, nblk]) == 1.0


@pytest.mark.parametrize("ctx,Hq,G", [((4999, 2048, 127, 255), 16, 2), ((20000, 131), 64, 8), ((2900, 1, 383), 16, 1)])
def test_fp8_decode_step_matches_oracle(cuda_ok, ctx, Hq, G):
    w = synth.Workload(name="t", kind="decode", B=len(ctx), Hq=Hq, G=G, ctx=tuple(ctx), seed=9090 + sum(ctx))
    l_cap = (max(ctx) + 1 + 127) // 128 * 128 + 128
    st = build_decode_state(w, l_cap)
    nb_cap = st["nb_cap"]
    f8 = pipeline.fp8_cache(st["k_cache"], st["v_cache"], nb_cap)
    for b in range(w.B):
        pipeline.fp8_quantize_sequence(st["k_cache"], st["v_cache"], f8, b, w.ctx[b], Hq)
    bufs = pipeline.decode_buffers(w.B, w.Hq, w.G, max(w.ctx), "cuda")
    out, lse, sel = pipeline.decode_step_fp8(st["q"], st["q_idx"], st["k_idx_new"], st["k_new"], st["v_new"],
                                             st["ctx"], st["k_cache"], st["v_cache"], st["tail"], st["pooled"], f8,
                                             bufs)
    torch.cuda.synchronize()
    for key in ("ws_append", "ws_select", "ws_attn"):
        s, info = msa_get_device_status(bufs[key])
        assert s == 0, (key, s, info)
    out, lse, sel = f32(host_bits(out)), lse.cpu().numpy(), sel.cpu().numpy()
    for b in range(w.B):
        Lb = w.ctx[b]
        t = np.array([Lb])
        ki = synth.decode_seq_np(w, b, "k_idx")
        pooled, _ = oracle.pool(ki, 128)
        qi = synth.decode_seq_np(w, b, "q_idx")
        q = synth.decode_seq_np(w, b, "q")
        kk = synth.decode_seq_np(w, b, "k")                  # [G, Lb + 1, d], the new token included
        vv = synth.decode_seq_np(w, b, "v")
        for g in range(w.G):
            ref, kth, _ = oracle.select_rows(t, qi[g][None], pooled[g])
            check_selection(sel[b, g][None], ref, kth, qi[g][None], pooled[g], t, label=f"fp8 decode ctx={ctx}")
            Kc, ks = oracle.fp8_quantize_blocks(kk[g], 128)
            Vc, vs = oracle.fp8_quantize_blocks(vv[g], 128)
            o, l, _ = oracle.attend_row_fp8(Lb, q[g * w.Hg:(g + 1) * w.Hg], Kc, Vc, ks, vs, kk[g], vv[g], sel[b, g])
            assert_close_attention(out[b, g * w.Hg:(g + 1) * w.Hg], o, f"fp8 decode b={b} g={g}")
            np.testing.assert_allclose(lse[b, g * w.Hg:(g + 1) * w.Hg], l, rtol=0, atol=2e-3)
            if (Lb + 1) % 128 == 0:                          # this step closed block Lb / 128
                j = Lb // 128
                got_c = f8["k_codes"][b, g, j * 128:(j + 1) * 128].cpu().numpy()
                assert (got_c == Kc[j * 128:(j + 1) * 128]).all()
                assert float(f8["v_scale"][b, g, j]) == float(vs[j])
