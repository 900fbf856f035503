"""Pins of the fp64 oracle against things other than itself (CPU only).

Every check uses an independent route: a numpy / torch library routine (mean, matmul,
lexsort, scaled_dot_product_attention, logsumexp), a closed form, an invariant of the
definition, or a constructed case whose answer is known by design. Sources for the
definition: the youmind article "MiniMax M3 sparse attention agents" (paragraph "The
mechanism that changes this", figure 1 caption, bullet "Predictable cost at every length":
Bk = 128, k = 16, 2,048 tokens) and the KuCoin flash "MiniMax launches MSA sparse attention
method and MiniMax-M3 model" (summary: GQA-based, exact softmax over the 16 blocks, exp-free
top-k).
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth
from tests.msa_check import compare_selection_row, sel_sorted_ok

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def make(N, Hq, G, d=128, dI=64, seed=1):
    w = synth.small_workload(N=N, Hq=Hq, G=G, d=d, dI=dI, seed=seed)
    return w, synth.prefill_inputs_np(w)


# ----------------------------------------------------------------------------- pooling
def test_pool_is_block_mean_and_tail_sum():
    rng = np.random.default_rng(0)
    N, G, dI, Bk = 37, 3, 8, 5
    bits = synth.f64_to_bf16_bits(rng.standard_normal((N, G, dI)))
    pooled, tail = oracle.pool(bits, Bk)
    ref = f32(bits)[: (N // Bk) * Bk].reshape(N // Bk, Bk, G, dI).mean(axis=1).transpose(1, 0, 2)
    assert pooled.shape == (G, N // Bk, dI)
    np.testing.assert_allclose(pooled, ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(tail, f32(bits)[(N // Bk) * Bk:].sum(axis=0), rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------- scores
def test_block_scores_match_matmul():
    rng = np.random.default_rng(1)
    dI, nb = 64, 50
    q = synth.f64_to_bf16_bits(rng.standard_normal(dI))
    pooled = rng.standard_normal((nb, dI))
    s = oracle.block_scores(q, pooled, 40)
    ref = pooled[:40] @ f32(q) / np.sqrt(dI)
    np.testing.assert_allclose(s, ref, rtol=1e-13, atol=1e-15)


# ----------------------------------------------------------------------------- selection
def _lexsort_select(s, c, topk):
    if c + 1 <= topk:
        return np.arange(c + 1)
    order = np.lexsort((np.arange(c), -s[:c]))     # primary: -s (score desc), secondary: id
    return np.sort(np.concatenate([order[: topk - 1], [c]]))


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_library_sort_with_ties(seed):
    rng = np.random.default_rng(seed)
    for c in [0, 1, 7, 14, 15, 16, 17, 40, 300]:
        # quantised scores force many exact ties
        s = np.round(rng.standard_normal(max(c, 1)) * 4) / 4
        sel, n, kth = oracle.select_from_scores(s, c, 16)
        ref = _lexsort_select(s, c, 16)
        assert n == len(ref)
        assert list(sel[:n]) == list(ref)
        assert all(v == -1 for v in sel[n:])
        assert sel_sorted_ok(sel)
        sel2, n2 = oracle.select_fullsort(s, c, 16)
        assert list(sel2) == list(sel)
        if c + 1 > 16:
            ranked = s[np.lexsort((np.arange(c), -s[:c]))]
            assert kth == ranked[14]
        else:
            assert np.isnan(kth)


def test_select_few_blocks_takes_all():
    for c in range(16):
        sel, n, _ = oracle.select_from_scores(np.zeros(max(c, 1)), c, 16)
        assert n == c + 1 and list(sel[: c + 1]) == list(range(c + 1))


def test_equal_scores_take_lowest_ids():
    # constant k_I (all pooled keys equal) or q_I = 0: every score ties -> {0..14, c}
    N, G, dI, Bk = 128 * 40, 1, 64, 128
    k_idx = np.full((N, G, dI), synth.f64_to_bf16_bits(np.array([0.75]))[0], np.uint16)
    pooled, _ = oracle.pool(k_idx, Bk)
    rng = np.random.default_rng(3)
    q = synth.f64_to_bf16_bits(rng.standard_normal((1, dI)))
    t = np.array([N - 1])
    sel, _, _ = oracle.select_rows(t, q, pooled[0], Bk, 16)
    assert list(sel[0]) == list(range(15)) + [39]
    zero_q = np.zeros((1, dI), np.uint16)
    k_rand = synth.f64_to_bf16_bits(rng.standard_normal((N, G, dI)))
    pooled2, _ = oracle.pool(k_rand, Bk)
    sel, _, _ = oracle.select_rows(t, zero_q, pooled2[0], Bk, 16)
    assert list(sel[0]) == list(range(15)) + [39]


def test_planted_blocks_are_selected():
    rng = np.random.default_rng(4)
    N, dI, Bk = 128 * 64, 64, 128
    k_idx = synth.f64_to_bf16_bits(rng.standard_normal((N, 1, dI)))
    q = synth.f64_to_bf16_bits(rng.standard_normal((1, dI)))
    planted = np.sort(rng.choice(63, 15, replace=False))
    qv = f32(q[0])
    for j in planted:                # add a large multiple of q_I to every key of the block
        k_idx[j * Bk:(j + 1) * Bk, 0] = synth.f64_to_bf16_bits(f32(k_idx[j * Bk:(j + 1) * Bk, 0]) + 6 * qv)
    pooled, _ = oracle.pool(k_idx, Bk)
    sel, _, _ = oracle.select_rows(np.array([N - 1]), q, pooled[0], Bk, 16)
    assert list(sel[0]) == list(planted) + [63]


def test_near_tie_rule():
    s = np.array([1.0, 0.5, 0.5 + 4e-6, 0.2])
    kth = 0.5 + 4e-6
    assert compare_selection_row([1, 3, -1], [2, 3, -1], s, kth) == (True, 2, 0)
    assert compare_selection_row([0, 3, -1], [2, 3, -1], s, kth)[0] is False
    assert compare_selection_row([2, 3, 3], [2, 3, -1], s, kth)[0] is False


def test_cancellation_window_only_when_the_kth_score_is_near_zero():
    # block 1 differs from the 15th score by 3e-6: outside 1e-5 * |kth|, inside 1e-5 * its
    # term magnitude (0.5). Accepted as a cancellation near-tie only when |kth| < 0.1 * 0.5.
    absscale = np.array([0.5, 0.5, 0.5, 0.5])
    s = np.array([1.0, 0.01 + 3e-6, 0.01, -1.0])
    assert compare_selection_row([1, 3, -1], [2, 3, -1], s, 0.01, absscale) == (True, 1, 1)
    s = np.array([1.0, 0.2 + 3e-6, 0.2, -1.0])
    assert compare_selection_row([1, 3, -1], [2, 3, -1], s, 0.2, absscale)[0] is False


def test_vectorised_row_validity():
    from tests.msa_check import sel_sorted_ok_rows
    rows = np.array([[0, 3, 9, -1], [0, 3, 3, -1], [0, -1, 2, -1], [5, 2, -1, -1], [1, 2, 3, 4], [-1, -1, -1, -1]])
    want = [sel_sorted_ok(r) for r in rows]
    assert list(sel_sorted_ok_rows(rows)) == want == [True, False, False, False, True, True]


# ----------------------------------------------------------------------------- attention
def _sdpa_masked(qf, kf, vf, mask):
    """torch fp64 attention. qf [H, T, d], kf/vf [U, d], mask [T, U] bool (True = attend)."""
    out = F.scaled_dot_product_attention(qf[None], kf[None, None].expand(1, qf.shape[0], -1, -1),
                                         vf[None, None].expand(1, qf.shape[0], -1, -1),
                                         attn_mask=mask[None, None])
    return out[0]


def test_dense_equivalence_when_all_blocks_fit():
    # c + 1 <= 16 for every query (N <= 2048): MSA reduces to dense causal GQA attention.
    w, x = make(N=300, Hq=4, G=2, seed=11)
    r = oracle.prefill(x, w.Hq, w.G)
    q = torch.from_numpy(f32(x["q"]))[0]            # [N, Hq, d]
    k = torch.from_numpy(f32(x["k"]))[0]            # [G, N, d]
    v = torch.from_numpy(f32(x["v"]))[0]
    Hg = w.Hq // w.G
    kk = k.repeat_interleave(Hg, dim=0)             # head h uses group h // Hg
    vv = v.repeat_interleave(Hg, dim=0)
    ref = F.scaled_dot_product_attention(q.permute(1, 0, 2)[None], kk[None], vv[None], is_causal=True)
    ref = ref[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(r["out"][0], ref, rtol=0, atol=1e-12)
    lse_ref = torch.logsumexp((q.permute(1, 0, 2) @ kk.transpose(1, 2)) / np.sqrt(128)
                              + torch.triu(torch.full((300, 300), -np.inf, dtype=torch.float64), 1),
                              dim=-1).permute(1, 0).numpy()
    np.testing.assert_allclose(r["lse"][0], lse_ref, rtol=0, atol=1e-11)
    od, _ = oracle.dense_gqa(x, w.Hq, w.G)
    np.testing.assert_allclose(od, r["out"], rtol=0, atol=1e-13)


def test_sparse_attention_matches_masked_sdpa():
    # small blocks (Bk = 4, k = 4) so that selection really drops blocks
    rng = np.random.default_rng(5)
    N, d, Bk, topk = 70, 32, 4, 4
    qb = synth.f64_to_bf16_bits(rng.standard_normal((N, 2, d)))
    kb = synth.f64_to_bf16_bits(rng.standard_normal((N, d)))
    vb = synth.f64_to_bf16_bits(rng.standard_normal((N, d)))
    sel = np.full((N, topk), -1, np.int32)
    for t in range(N):
        c = t // Bk
        cand = rng.permutation(c)[: topk - 1] if c + 1 > topk else np.arange(c)
        ids = np.sort(np.concatenate([cand, [c]]))
        sel[t, : len(ids)] = ids
    o, lse, nk = oracle.attend_rows(np.arange(N), qb, kb, vb, sel, Bk, topk)
    mask = np.zeros((N, N), bool)
    for t in range(N):
        for u in range(t + 1):
            mask[t, u] = (u // Bk) in set(sel[t][sel[t] >= 0])
    ref = _sdpa_masked(torch.from_numpy(f32(qb)).permute(1, 0, 2), torch.from_numpy(f32(kb)),
                       torch.from_numpy(f32(vb)), torch.from_numpy(mask))
    np.testing.assert_allclose(o, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    assert list(nk) == list(mask.sum(1))


def test_constant_v_gives_v():
    w, x = make(N=2600, Hq=4, G=1, seed=12)
    x["v"][:] = synth.f64_to_bf16_bits(np.array([-1.375]))[0]
    t = np.array([0, 1, 127, 128, 2047, 2048, 2599])
    pooled, _ = oracle.pool(x["k_idx"][0], 128)
    sel, _, _ = oracle.select_rows(t, x["q_idx"][0, t, 0], pooled[0])
    o, _, _ = oracle.attend_rows(t, x["q"][0, t], x["k"][0, 0], x["v"][0, 0], sel)
    np.testing.assert_allclose(o, -1.375, rtol=0, atol=1e-13)


def test_permutation_inside_selected_block_is_invariant():
    w, x = make(N=128 * 24, Hq=4, G=1, seed=13)
    t = np.arange(128 * 23, 128 * 24)
    r0 = _rows(x, t)
    # the non-diagonal block that the most queries of the last block selected
    counts = np.bincount(r0["sel"][r0["sel"] >= 0].ravel(), minlength=24)[:23]
    j = int(np.argmax(counts))
    assert counts[j] > 0
    perm = np.random.default_rng(0).permutation(128) + 128 * j
    y = {k: v.copy() for k, v in x.items()}
    y["k"][0, 0, 128 * j:128 * (j + 1)] = x["k"][0, 0, perm]
    y["v"][0, 0, 128 * j:128 * (j + 1)] = x["v"][0, 0, perm]
    y["k_idx"][0, 128 * j:128 * (j + 1)] = x["k_idx"][0, perm]
    r1 = _rows(y, t)
    assert (r0["sel"] == r1["sel"]).all()
    np.testing.assert_allclose(r1["o"], r0["o"], rtol=0, atol=1e-13)


def _rows(x, t):
    pooled, _ = oracle.pool(x["k_idx"][0], 128)
    sel, kth, _ = oracle.select_rows(t, x["q_idx"][0, t, 0], pooled[0])
    o, lse, nk = oracle.attend_rows(t, x["q"][0, t], x["k"][0, 0], x["v"][0, 0], sel)
    return {"sel": sel, "o": o, "lse": lse, "nk": nk}


# ----------------------------------------------------------------------------- key counts
def closed_form_total_keys(N, Bk=128, k=16):
    """Sum over queries of attended keys: t < k*Bk attend t+1 keys; later queries at offset
    i of their block attend (k-1)*Bk + i + 1 keys."""
    assert N % Bk == 0 and N >= k * Bk
    head = (k * Bk) * (k * Bk + 1) // 2
    per_block = Bk * (k - 1) * Bk + Bk * (Bk + 1) // 2
    return head + (N // Bk - k) * per_block


def test_closed_form_key_counts_golden():
    with open(os.path.join(GOLDEN, "key_counts.json")) as f:
        gold = json.load(f)
    for n, total in gold["totals"].items():
        assert closed_form_total_keys(int(n)) == total


def test_oracle_key_counts_match_closed_form():
    w, x = make(N=4096, Hq=4, G=1, seed=14)
    x["q"] = x["q"][:, :, :1]          # one head is enough to count keys
    pooled, _ = oracle.pool(x["k_idx"][0], 128)
    t = np.arange(4096)
    sel, _, _ = oracle.select_rows(t, x["q_idx"][0, :, 0], pooled[0])
    _, _, nk = oracle.attend_rows(t, x["q"][0], x["k"][0, 0], x["v"][0, 0], sel)
    assert int(nk.sum()) == closed_form_total_keys(4096) == 6162432
    for tt in [2048, 2049, 3000, 4095]:
        assert nk[tt] == 1920 + tt % 128 + 1


# ----------------------------------------------------------------------------- top-k of score rows
# The selection step on its own (KuCoin flash "MiniMax launches MSA sparse attention method and
# MiniMax-M3 model", "ME AI News" paragraph: exp-free top-k, compared with torch.topk).
@pytest.mark.parametrize("seed", [0, 1])
def test_topk_rows_match_lexsort_with_ties(seed):
    rng = np.random.default_rng(seed)
    rows, n, k = 40, 97, 15
    s = (np.round(rng.standard_normal((rows, n)) * 2.0) / 2.0).astype(np.float32)   # many exact ties
    got = oracle.topk_rows(s, k)
    cols = np.arange(n)
    for i in range(rows):
        want = np.lexsort((cols, -s[i].astype(np.float64)))[:k]     # score desc, then column asc
        assert got[i].tolist() == want.tolist()


def test_topk_rows_distinct_values_match_torch_topk():
    g = torch.Generator().manual_seed(5)
    s = torch.randn(64, 1024, generator=g)
    want = torch.topk(s, 16, dim=1, largest=True, sorted=True).indices.numpy()
    assert (oracle.topk_rows(s.numpy(), 16) == want).all()


def test_topk_rows_special_values():
    nan, inf = float("nan"), float("inf")
    row = np.array([[1.0, nan, -inf, inf, -0.0, 0.0, nan, -1.0, 2.0]], np.float32)
    # NaNs first (lower column first), then +inf, 2, 1, the two zeros by column, -1, -inf
    assert oracle.topk_rows(row, 9)[0].tolist() == [1, 6, 3, 8, 0, 4, 5, 7, 2]
    assert oracle.topk_rows(row, 3)[0].tolist() == [1, 6, 3]


def test_topk_rows_constant_and_descending_rows():
    assert (oracle.topk_rows(np.full((3, 50), 0.25, np.float32), 16) == np.arange(16)).all()
    desc = -np.arange(33, dtype=np.float32)[None, :].repeat(2, axis=0)
    assert (oracle.topk_rows(desc, 16) == np.arange(16)).all()
    asc = np.arange(33, dtype=np.float32)[None, :]
    assert oracle.topk_rows(asc, 4)[0].tolist() == [32, 31, 30, 29]


# ----------------------------------------------------------------------------- FP8 (e4m3) key-value cache
# The compressed cache of the decode variant (KuCoin flash "MiniMax launches MSA sparse attention
# method and MiniMax-M3 model", "ME AI News" paragraph: the SM100 kernel also takes FP8 inputs).
def test_e4m3_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_to_f64(codes.numpy())
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert (got[ok] == want[ok]).all() and (np.signbit(got[ok]) == np.signbit(want[ok])).all()


def test_e4m3_encode_matches_torch_rounding():
    # every finite code, every midpoint between neighbouring codes (the ties), random values;
    # |x| <= 464, where torch's cast and a saturating one agree
    grid = oracle.e4m3_to_f64(np.arange(127, dtype=np.uint8))
    mids = (grid[:-1] + grid[1:]) / 2
    rng = np.random.default_rng(0)
    rnd = rng.uniform(-464, 464, 20000) * 10.0 ** rng.uniform(-6, 0, 20000)
    x = np.concatenate([grid, -grid[1:], mids, -mids, rnd, [464.0, -464.0]]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (oracle.e4m3_from_f32(x) == want).all()


def test_e4m3_encodes_nan_as_nan():
    x = np.array([np.nan, -np.nan], np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_from_f32(x)
    assert (got == want).all() and got.tolist() == [0x7F, 0xFF]
    assert np.isnan(oracle.e4m3_to_f64(got)).all()


def test_e4m3_saturates_beyond_448():
    x = np.array([448.5, 463.9, 465.0, 1e6, 3e38, -500.0], np.float32)
    assert oracle.e4m3_from_f32(x).tolist() == [126, 126, 126, 126, 126, 254]


def test_fp8_block_quantisation_bounds():
    rng = np.random.default_rng(1)
    xb = synth.f64_to_bf16_bits(rng.standard_normal((300, 128)) * 3.0)
    codes, scales = oracle.fp8_quantize_blocks(xb, 128)
    assert len(scales) == 3
    x = f32(xb)
    for j in range(3):
        blk = x[j * 128:(j + 1) * 128]
        amax = np.abs(blk).max()
        assert abs(scales[j] - amax / 448.0) <= amax / 448.0 * 2.0 ** -23
        cv = oracle.e4m3_to_f64(codes[j * 128:(j + 1) * 128])
        assert np.abs(cv).max() == 448.0                    # the largest magnitude maps to 448
        # 3 mantissa bits: half a unit in the last place is at most 2^-4 of |x|; the subnormal
        # spacing 2^-9 leaves at most 2^-10 absolute; both in units of the scale
        err = np.abs(cv * float(scales[j]) - blk)
        assert (err <= (np.abs(blk) * 2.0 ** -4 + 2.0 ** -10 * float(scales[j])) * (1 + 1e-6)).all()
    zc, zs = oracle.fp8_quantize_blocks(np.zeros((5, 128), np.uint16), 128)
    assert zs.tolist() == [1.0] and not zc.any()


def test_fp8_quantisation_commutes_with_powers_of_two():
    rng = np.random.default_rng(2)
    xb = synth.f64_to_bf16_bits(rng.standard_normal((128, 128)))
    c1, s1 = oracle.fp8_quantize_blocks(xb)
    c2, s2 = oracle.fp8_quantize_blocks(synth.f64_to_bf16_bits(f32(xb) * 2.0 ** 5))
    assert (c1 == c2).all() and s2[0] == s1[0] * 2.0 ** 5


def test_fp8_attention_equals_bf16_attention_on_a_representable_cache():
    # closed blocks hold exactly code * 2^e with a +-448 in every block, so quantisation gives
    # back the same codes and scales 2^e, and attention over the FP8 cache must equal step 4 on
    # the bf16 cache bit for bit; the open block holds arbitrary bf16 values, which only the
    # bf16 rows carry exactly
    rng = np.random.default_rng(3)
    L, d, Bk, Hg = 128 * 20 + 17, 128, 128, 4
    nb_closed = L // Bk
    finite = np.array([c for c in range(1, 255) if c not in (127, 128)], np.uint8)

    def cache():
        codes = rng.choice(finite, size=(L, d))
        vals = oracle.e4m3_to_f64(codes)
        for j in range(nb_closed):
            vals[j * Bk, 0] = 448.0
            vals[j * Bk:(j + 1) * Bk] *= 2.0 ** int(rng.integers(-9, -3))
        vals[nb_closed * Bk:] = rng.standard_normal((L - nb_closed * Bk, d))
        return synth.f64_to_bf16_bits(vals)

    K, V = cache(), cache()
    Kc, ks = oracle.fp8_quantize_blocks(K, Bk)
    Vc, vs = oracle.fp8_quantize_blocks(V, Bk)
    assert (oracle.e4m3_to_f64(Kc[:nb_closed * Bk]) * np.repeat(ks[:nb_closed], Bk)[:, None]
            == f32(K[:nb_closed * Bk])).all()
    q = synth.f64_to_bf16_bits(rng.standard_normal((Hg, d)))
    t = L - 1
    sel = np.array([0, 1, 2, 3, 5, 6, 7, 9, 10, 11, 13, 14, 15, 17, 19, t // Bk], np.int32)
    o8, l8, n8 = oracle.attend_row_fp8(t, q, Kc, Vc, ks, vs, K, V, sel, Bk)
    o, l, n = oracle.attend_rows(np.array([t]), q[None], K, V, sel[None], Bk)
    assert n8 == n[0] == 15 * Bk + (t % Bk) + 1
    assert np.array_equal(o8, o[0]) and np.array_equal(l8, l[0])


# ----------------------------------------------------------------------------- step 4, gradient
# The main branch's backward pass (dQ, dK, dV over the selected blocks, the selection held
# fixed), the oracle of a later kernel: torch fp64 autograd of the equivalent masked dense
# attention, and identities of the softmax gradient.
def _grad_case(seed, N=150, Hg=2, d=32, Bk=16, k=4, grid=None):
    rng = np.random.default_rng(seed)
    vals = lambda shape: (np.round(rng.standard_normal(shape) * 16) / 16).clip(-4, 4) if grid else rng.standard_normal(shape)
    q = synth.f64_to_bf16_bits(vals((N, Hg, d)))
    K = synth.f64_to_bf16_bits(vals((N, d)))
    V = synth.f64_to_bf16_bits(vals((N, d)))
    sel = np.full((N, k), -1, np.int32)
    for t in range(N):
        c = t // Bk
        ids = list(range(c + 1)) if c + 1 <= k else sorted(rng.choice(c, k - 1, replace=False).tolist()) + [c]
        sel[t, :len(ids)] = ids
    dO = rng.standard_normal((N, Hg, d))
    return q, K, V, sel, dO


def test_attention_grad_matches_torch_autograd():
    N, Hg, d, Bk, k = 150, 2, 32, 16, 4
    q, K, V, sel, dO = _grad_case(0, N, Hg, d, Bk, k)
    dQ, dK, dV = oracle.attend_grad(np.arange(N), q, K, V, sel, dO, Bk)
    qt = torch.tensor(f32(q), requires_grad=True)
    kt = torch.tensor(f32(K), requires_grad=True)
    vt = torch.tensor(f32(V), requires_grad=True)
    u = torch.arange(N)
    mask = (u[None, :] <= u[:, None]) & torch.tensor(
        [[(j // Bk) in set(sel[t][sel[t] >= 0].tolist()) for j in range(N)] for t in range(N)])
    z = torch.einsum("thd,ud->thu", qt, kt) / np.sqrt(d)
    z = z.masked_fill(~mask[:, None, :], float("-inf"))
    o = torch.einsum("thu,ud->thd", torch.softmax(z, dim=-1), vt)
    (o * torch.tensor(dO)).sum().backward()
    np.testing.assert_allclose(dQ, qt.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dK, kt.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dV, vt.grad.numpy(), rtol=0, atol=1e-10)


def test_attention_grad_identities():
    N, Hg, d, Bk, k = 120, 2, 32, 16, 4
    q, K, V, sel, dO = _grad_case(1, N, Hg, d, Bk, k, grid=True)
    t = np.arange(N)
    dQ, dK, dV = oracle.attend_grad(t, q, K, V, sel, dO, Bk)
    # the softmax gradient sums to zero over a row's keys, so the keys' gradients sum to zero
    assert np.abs(dK.sum(axis=0)).max() < 1e-9
    # shifting every key by one vector shifts all of a row's scores equally: nothing changes
    K2 = synth.f64_to_bf16_bits(f32(K) + 0.25)
    assert (f32(K2) == f32(K) + 0.25).all()                # exact on the 1/16 grid
    dQ2, dK2, dV2 = oracle.attend_grad(t, q, K2, V, sel, dO, Bk)
    for a, b in ((dQ, dQ2), (dK, dK2), (dV, dV2)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-9)
    # a query that attends one key (position 0): dQ = 0, dK_0 = 0, dV_0 = dO summed over heads
    g0Q, g0K, g0V = oracle.attend_grad(np.array([0]), q[:1], K, V, sel[:1], dO[:1], Bk)
    assert not g0Q.any() and not g0K.any()
    np.testing.assert_array_equal(g0V[0], dO[0].sum(axis=0))
    assert not g0V[1:].any()


# ----------------------------------------------------------------------------- chunked prefill
@pytest.mark.parametrize("P,n", [(0, 300), (1000, 700), (1700, 1), (128 * 20, 128 * 3 + 5)])
def test_chunk_rows_equal_whole_prefill_rows(P, n):
    # a chunk at positions P .. P + n - 1 against the sequence so far is rows P .. P + n - 1 of a
    # prefill of the whole sequence (the definition is per query position)
    w, x = make(N=P + n, Hq=4, G=2, seed=P + n)
    full = oracle.prefill(x, w.Hq, w.G)
    r = oracle.prefill_chunk(x["q"][0, P:], x["q_idx"][0, P:], x["k_idx"][0], x["k"][0], x["v"][0], P, w.Hq, w.G)
    assert (r["sel"] == full["sel"][0, P:]).all()
    np.testing.assert_array_equal(r["kth"], full["kth"][0, P:])
    np.testing.assert_array_equal(r["out"], full["out"][0, P:])
    np.testing.assert_array_equal(r["lse"], full["lse"][0, P:])


def test_chunk_reduces_to_dense_causal_attention_when_every_block_fits():
    # P + n <= 2048: every query takes every block, so a chunk is dense causal GQA attention over
    # positions 0 .. t (torch fp64 SDPA with an explicit mask on the chunk's rows)
    P, n = 900, 400
    w, x = make(N=P + n, Hq=4, G=2, seed=5)
    r = oracle.prefill_chunk(x["q"][0, P:], x["q_idx"][0, P:], x["k_idx"][0], x["k"][0], x["v"][0], P, w.Hq, w.G)
    q = torch.from_numpy(f32(x["q"][0, P:]))                   # [n, Hq, d]
    Hg = w.Hq // w.G
    t = torch.arange(P, P + n)[:, None]
    mask = torch.arange(P + n)[None, :] <= t                 # [n, P + n]
    for h in range(w.Hq):
        kf = torch.from_numpy(f32(x["k"][0, h // Hg]))
        vf = torch.from_numpy(f32(x["v"][0, h // Hg]))
        ref = _sdpa_masked(q[:, h][None], kf, vf, mask)[0]
        np.testing.assert_allclose(r["out"][:, h], ref.numpy(), rtol=0, atol=1e-12)
