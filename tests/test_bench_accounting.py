"""The benchmark's work counts (the numerators of its roofline fractions) against the golden
key counts and closed forms, on the CPU. Sources: youmind article "MiniMax M3 sparse attention
agents", bullet "Predictable cost at every length" (Bk = 128, k = 16: 2,048 key-value tokens
per query and GQA group)."""
import json
import os

import pytest

import bench

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "key_counts.json")


def test_attended_pairs_match_golden_totals():
    totals = json.load(open(GOLDEN))["totals"]
    for n, want in totals.items():
        assert bench.attended_pairs(int(n)) == want


@pytest.mark.parametrize("N,Bk,k", [(1000, 16, 4), (77, 8, 3), (64, 16, 4)])
def test_attended_pairs_by_explicit_key_sets(N, Bk, k):
    # every query keeps its own block plus up to k-1 full past blocks: count the keys of an
    # explicit selection (the first k-1 past blocks) one by one
    total = 0
    for t in range(N):
        c = t // Bk
        sel = set(range(c + 1)) if c + 1 <= k else set(range(k - 1)) | {c}
        total += sum(1 for u in range(t + 1) if u // Bk in sel)
    assert bench.attended_pairs(N, Bk, k) == total


def test_prefill_flop_counts():
    w = bench.PREFILL
    assert (w.N, w.Hq, w.G, w.d, w.dI) == (131072, 64, 8, 128, 64)
    assert bench.prefill_main_flops(w) == 4 * 128 * 64 * 258146304          # 8.459e12
    nb = 131072 // 128                                                        # 1,024 blocks
    assert bench.prefill_index_flops(w) == 2 * 64 * 8 * 128 * (nb * (nb - 1) // 2)   # 6.87e10


def test_prefill_index_flops_ragged_tail_by_enumeration():
    import dataclasses
    w = dataclasses.replace(bench.PREFILL, N=128 * 5 + 37)
    cand = sum(t // 128 for t in range(w.N))
    assert bench.prefill_index_flops(w) == 2 * 64 * w.G * w.B * cand


def test_decode_step_bytes_closed_form():
    w = bench.DECODE
    assert (w.B, w.Hq, w.G) == (16, 64, 8) and set(w.ctx) == {131072}
    d = bench.decode_step_bytes(w)
    per_bg_pooled = 1024 * 64 * 4                          # every fully-past block's pooled key
    per_bg_kv = (15 * 128 + 1) * 128 * 2 * 2               # 15 full blocks + the new token, K and V
    small = 16 * (64 * 128 * 2 * 2 + 8 * 64 * 2 * 2 + 8 * 128 * 2 * 2 * 2 + 8 * 64 * 4 * 2 + 8 * 16 * 4)
    assert d["pooled"] == 128 * per_bg_pooled
    assert d["kv"] == 128 * per_bg_kv
    assert d["total"] == 128 * (per_bg_pooled + per_bg_kv) + small == 160210944


def test_partial_rows_by_enumeration():
    # one partial per (token, head, selected block): the own block plus min(c, k - 1) past ones
    import dataclasses
    for N in (77, 128 * 3, 128 * 20 + 5):
        w = dataclasses.replace(bench.PREFILL, N=N, Hq=4, G=1)
        want = sum(min(t // 128, 15) + 1 for t in range(N)) * 4
        assert bench.prefill_main_bytes(w)["partial_rows"] == want
    w = bench.PREFILL
    rows = bench.prefill_main_bytes(w)["partial_rows"]
    assert rows == (128 * sum(c + 1 for c in range(16)) + (131072 - 2048) * 16) * 64 == 133234688


def test_captured_traffic_is_dropped_when_sources_change(monkeypatch):
    files = ["select.cu"]
    good = {"sources": files, "sha16": bench.source_sha16(files), "bytes": 1000, "note": "n", "profile": "p.md"}
    monkeypatch.setitem(bench.CAPTURES, "probe", good)
    assert bench.captured_traffic("probe", 2.0)[0] == 2000
    monkeypatch.setitem(bench.CAPTURES, "probe", dict(good, sha16="0" * 16))
    got, why = bench.captured_traffic("probe", 2.0)
    assert got is None and "changed" in why
    assert bench.captured_traffic("absent", 1.0)[0] is None


def test_recorded_captures_are_close_to_their_models():
    # every recorded capture: traffic within a few percent above the model it is scaled by
    c = bench.CAPTURES
    if "decode_step" in c:
        assert 1.0 <= c["decode_step"]["bytes"] / c["decode_step"]["algorithmic_bytes"] < 1.05
    if "prefill_main" in c:
        assert 0.9 <= c["prefill_main"]["bytes"] / c["prefill_main"]["model_bytes"] < 1.2
    if "attn_prefill" in c:
        assert 0.9 <= c["attn_prefill"]["bytes"] / c["attn_prefill"]["model_bytes"] < 1.2
    if "topk_rows" in c:
        rows = c["topk_rows"]["rows"]
        # reads equal the scores; some of the ids' writes can still be dirty in L2 when the kernel ends
        assert 0.99 <= c["topk_rows"]["bytes"] / (rows * 1024 * 4 + rows * 15 * 4) < 1.02


def test_attention_byte_model_is_part_of_the_call_model():
    m = bench.prefill_main_bytes(bench.PREFILL)
    # the call = attention + inverted index + combine: attention writes the partials once, the
    # combine reads them back
    assert m["partials"] < m["attn_model"] < m["model"] - m["partials"]
    assert m["partial_rows"] == 133234688


def test_fp8_decode_step_bytes_closed_form():
    w = bench.DECODE
    d8, d = bench.decode_step_bytes_fp8(w), bench.decode_step_bytes(w)
    per_bg_kv = 15 * (128 * 128 * 1 * 2 + 2 * 4) + 1 * 128 * 2 * 2   # e4m3 K and V + scales, own block bf16
    assert d8["kv"] == 128 * per_bg_kv
    assert d8["pooled"] == d["pooled"] and d8["small"] == d["small"]
    assert d8["total"] == 97311744


def test_kernel_means_per_step():
    recs = [("split_keys", 0.01), ("select_prefill", 1.0), ("attn_prefill", 14.0), ("combine", 6.0),
            ("split_keys", 0.03), ("select_prefill", 1.2), ("attn_prefill", 16.0), ("combine", 6.0),
            ("inverted_index", 0.1), ("inverted_index", 0.3)]
    k = bench.kernel_means(recs, 2)
    assert k["attn_prefill"] == {"ms": 15.0, "launches": 1.0}
    assert abs(k["split_keys"]["ms"] - 0.02) < 1e-12 and k["inverted_index"]["launches"] == 1.0
    assert set(k) == {"split_keys", "select_prefill", "attn_prefill", "combine", "inverted_index"}
