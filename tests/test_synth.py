"""The seeded input generator: determinism, distributions, canonical layout."""
import numpy as np

import oracle
import synth


def test_streams_are_deterministic_and_independent():
    wl = synth.WORKLOADS["tiny"]
    a = synth.expert_blob(wl, 0, 3)
    b = synth.expert_blob(wl, 0, 3)
    c = synth.expert_blob(wl, 0, 4)
    d = synth.expert_blob(wl, 1, 3)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    many = synth.expert_blobs(wl, 0, 2, 4)
    assert np.array_equal(many[1], a)


def test_distributions_match_recipe():
    wl = synth.WORKLOADS["layer"]
    blob = synth.expert_blob(wl, 0, 0)
    H, I = wl.hidden, wl.inter
    cb = I * H // 2
    codes = np.frombuffer(blob[:cb].tobytes(), dtype=np.uint8)
    nib = np.concatenate([codes & 0xF, codes >> 4])
    counts = np.bincount(nib, minlength=16)
    assert counts.min() > 0.9 * nib.size / 16 and counts.max() < 1.1 * nib.size / 16
    ng = I * H // 64
    s = oracle.bf16_to_f64(np.frombuffer(blob[cb: cb + 2 * ng].tobytes(), dtype="<u2"))
    b = oracle.bf16_to_f64(np.frombuffer(blob[cb + 2 * ng: cb + 4 * ng].tobytes(), dtype="<u2"))
    assert s.min() >= 0.005 - 1e-4 and s.max() <= 0.02 + 1e-4 and abs(s.mean() - 0.0125) < 1e-4
    assert b.min() >= -0.1 - 1e-3 and b.max() <= 0.1 + 1e-3 and abs(b.mean()) < 2e-3
    x = oracle.bf16_to_f64(synth.token(wl, 0))
    assert abs(x.mean()) < 0.06 and abs(x.std() - 1.0) < 0.05
    wr = oracle.bf16_to_f64(synth.router_weight(wl, 0))
    assert abs(wr.std() - 0.02) < 5e-4
    nw = oracle.bf16_to_f64(synth.norm_weight(synth.WORKLOADS["stack4"], 0))
    assert abs(nw.mean() - 1.0) < 2e-3 and abs(nw.std() - 0.02) < 3e-3


def test_bf16_rounding_agrees_with_independent_implementation():
    rng = np.random.default_rng(0)
    vals = rng.standard_normal(20000) * 10.0 ** rng.integers(-40, 40, 20000)
    vals = np.concatenate([vals, [1 + 2.0**-8, 1 + 3 * 2.0**-8, 2.0**-133, 1.5 * 2.0**-133, 3e38, 4e38, -0.0]])
    for v in vals:
        assert synth.double_to_bf16(v) == oracle.round_bf16(v)


def test_zipf_bias_is_a_permutation_of_log_ranks():
    wl = synth.WORKLOADS["batched"]
    b = synth.zipf_bias(wl, 0)
    ranks = np.exp(-b.astype(np.float64) / wl.zipf)
    assert np.allclose(np.sort(ranks), np.arange(1, wl.n_experts + 1), rtol=1e-5)
    assert synth.zipf_bias(synth.WORKLOADS["layer"], 0) is None
