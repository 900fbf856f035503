"""Seeded input generator: determinism, host/device equality, distribution (CPU only)."""
import numpy as np
import torch

import synth


def test_host_and_torch_generators_agree_bit_for_bit():
    a = synth.normal_bf16(99, synth.STREAM_K, (3, 1000))
    b = synth.normal_bf16_torch(99, synth.STREAM_K, 3000, "cpu").view(torch.int16).numpy()
    assert (a.ravel() == b.view(np.uint16)).all()
    # index-addressed subsets equal the corresponding slice of the whole tensor
    idx = np.array([0, 5, 2999, 1234], dtype=np.uint64)
    assert (synth.normal_bf16_at(99, synth.STREAM_K, idx) == a.ravel()[idx.astype(int)]).all()
    # offsets: start parameter continues the counter
    c = synth.normal_bf16(99, synth.STREAM_K, (1000,), start=2000)
    assert (c == a.ravel()[2000:]).all()


def test_streams_and_seeds_differ():
    a = synth.normal_bf16(1, 0, (4096,))
    assert not (a == synth.normal_bf16(1, 1, (4096,))).all()
    assert not (a == synth.normal_bf16(2, 0, (4096,))).all()


def test_distribution_is_standard_normal():
    x = synth.bf16_bits_to_f32(synth.normal_bf16(5, 0, (1 << 21,))).astype(np.float64)
    assert abs(x.mean()) < 3e-3 and abs(x.std() - 1) < 3e-3
    # quantiles of N(0,1): P(x < 1) = 0.8413, P(x < -2) = 0.02275
    assert abs((x < 1).mean() - 0.8413) < 2e-3 and abs((x < -2).mean() - 0.02275) < 1e-3


def test_bf16_rounding_nearest_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.0
    assert synth.f64_to_bf16_bits(np.array([1.0 + 2 ** -8]))[0] == 0x3F80
    assert synth.f64_to_bf16_bits(np.array([1.0 + 3 * 2 ** -8]))[0] == 0x3F82
    f = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (synth.f32_to_bf16_bits(f) == ref).all()
    assert (synth.f32_to_bf16_torch(torch.from_numpy(f)).view(torch.int16).numpy().view(np.uint16) == ref).all()


def test_planted_workload_structure():
    w = synth.Workload(name="t", kind="prefill", B=1, N=128 * 32, Hq=8, G=2, seed=3, planted=4)
    x = synth.prefill_inputs_np(w)
    shift, blocks = synth.plant_plan(w, x["q_idx"])
    assert np.allclose(np.linalg.norm(shift, axis=-1), 2.0, atol=1e-6)
    for (b, g), blks in blocks.items():
        assert len(set(blks)) == 4 and max(blks) < 31
    xt = synth.prefill_inputs_torch(w, "cpu")
    for name in x:
        assert (xt[name].view(torch.int16).numpy().view(np.uint16) == x[name]).all(), name


def test_decode_sequence_subsets():
    w = synth.Workload(name="d", kind="decode", B=2, Hq=8, G=2, ctx=(300, 257), seed=9)
    k_all = synth.decode_seq_np(w, 1, "k")                     # [G, L, d]
    assert k_all.shape == (2, 258, 128)
    assert (synth.decode_seq_np(w, 1, "k", 100, 200, g=1) == k_all[1, 100:200]).all()
    ki = synth.decode_seq_np(w, 0, "k_idx")                    # [L, G, dI]
    assert (synth.decode_seq_np(w, 0, "k_idx", 10, 20, g=1) == ki[10:20, 1]).all()
    kt = synth.decode_seq_torch(w, 1, "k", "cpu").view(torch.int16).numpy().view(np.uint16)
    assert (kt == k_all).all()
