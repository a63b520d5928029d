"""The seeded input generator (synth.py) follows its stated recipe, on CPU.

The generator holds none of the layer's arithmetic; these tests check the
value distributions, the seeds, the bf16 rounding and the routing skew that
the workloads are defined with, so that a changed draw is caught before it
changes every parity case and bench number at once.
"""
import dataclasses

import numpy as np

import synth


def test_workload_seeds_and_shapes():
    w = synth.WORKLOADS
    assert [w[n].seed for n in ("tiny", "decode1", "decode32", "prefill4096", "latent16")] == \
        [1000, 1001, 1002, 1003, 1004]
    assert (w["decode1"].T, w["decode1"].H, w["decode1"].I, w["decode1"].E, w["decode1"].k) == \
        (1, 8192, 2048, 512, 10)
    assert w["latent16"].W == 2048 and w["decode1"].W == 8192


def test_bf16_rounding_is_nearest_even():
    # halfway cases between neighbouring bf16 values go to the even one
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -8 + 2.0 ** -20],
                 np.float32)
    assert synth.f32_to_bf16_bits(v).tolist() == [0x3F80, 0x3F82, 0xBF80, 0x3F81]
    # values already in bf16 come back unchanged
    x = synth.bf16_bits_to_f32(np.arange(0x3F00, 0x4100, dtype=np.uint16))
    assert np.array_equal(synth.f32_to_bf16_bits(x), np.arange(0x3F00, 0x4100, dtype=np.uint16))


def test_dense_value_distributions():
    w = dataclasses.replace(synth.WORKLOADS["decode1"], T=64, E=64)
    d = synth.dense_inputs(w)
    x = synth.bf16_bits_to_f32(d["x"]).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    for name in ("w_router", "ws_gate", "ws_up", "ws_down", "w_sgate"):
        v = synth.bf16_bits_to_f32(d[name]).astype(np.float64)
        assert abs(v.std() / 0.02 - 1.0) < 0.02, name
        assert abs(v.mean()) < 0.002, name
    # every stream is its own: two matrices of the same shape differ
    assert not np.array_equal(d["ws_gate"], d["ws_up"])


def test_expert_codes_and_scales_are_uniform():
    q, s = synth.expert_matrix(1001, "gate", 7, 256, 2048)
    assert q.shape == (256, 1024) and s.shape == (256, 64)
    codes = np.concatenate([q & 0xF, q >> 4]).ravel()
    f = np.bincount(codes, minlength=16) / codes.size
    assert np.all(np.abs(f - 1 / 16) < 0.005)
    assert s.min() == 120 and s.max() == 127
    fs = np.bincount(s.ravel() - 120, minlength=8) / s.size
    assert np.all(np.abs(fs - 1 / 8) < 0.02)
    # one expert's matrix regenerates on its own, and experts differ
    assert np.array_equal(q, synth.expert_matrix(1001, "gate", 7, 256, 2048)[0])
    assert not np.array_equal(q, synth.expert_matrix(1001, "gate", 8, 256, 2048)[0])


def test_decode32_skew_hot_set():
    w = dataclasses.replace(synth.WORKLOADS["decode32"], T=2000)
    sets = synth.skew_sets(w)
    skewed = [S for S in sets if len(S)]
    assert abs(len(skewed) / w.T - 0.6) < 0.04
    pool = set(np.concatenate(skewed).tolist())
    assert len(pool) <= 64
    assert all(len(set(S.tolist())) == w.k for S in skewed)


def test_prefill_skew_is_zipf_over_all_experts():
    w = dataclasses.replace(synth.WORKLOADS["prefill4096"], T=1024)
    sets = synth.skew_sets(w)
    assert all(len(S) == w.k and len(set(S.tolist())) == w.k for S in sets)
    counts = np.bincount(np.concatenate(sets), minlength=w.E)
    # rank^-1.1 weights: the most chosen expert far above the median one
    assert counts.max() > 10 * np.median(counts)


def test_skew_boost_lifts_the_preferred_logits_by_about_8():
    w = dataclasses.replace(synth.WORKLOADS["decode32"], T=256, H=2048, E=128)
    d = synth.dense_inputs(w)
    plain = synth.dense_inputs(dataclasses.replace(w, skew="none"))
    wr = synth.bf16_bits_to_f32(d["w_router"]).astype(np.float64)
    lift = (synth.bf16_bits_to_f32(d["x"]).astype(np.float64)
            - synth.bf16_bits_to_f32(plain["x"]).astype(np.float64)) @ wr.T
    got = [lift[t, S].mean() for t, S in enumerate(synth.skew_sets(w)) if len(S)]
    assert len(got) > 100
    assert abs(np.mean(got) - 8.0) < 0.5
