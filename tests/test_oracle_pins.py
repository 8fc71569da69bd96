"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test ties the oracle to the pages (byte counts), to a hand derivation, to a
closed form, to an invariant of the mathematics or to brute force, so that a
dropped term, a wrong sign, index or group, a transposed operand or a swapped
gate/up would fail at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth
from canon import bf16_bits, make_blob

silu = lambda t: t / (1.0 + math.exp(-t))


# ----------------------------------------------------------------------------- byte counts


def test_blob_bytes_match_pages(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "expert_bytes.json")))
    H, I = fx["hidden"], fx["inter"]
    assert oracle.blob_bytes(H, I, 4) == fx["blob_bytes_4bit"]
    assert oracle.blob_bytes(H, I, 2) == fx["blob_bytes_2bit"]
    assert fx["blob_bytes_4bit"] == fx["pages_mb_4bit"] * 2**20
    # 60 layers x (512 routed + 1 shared) experts plus the non-expert weights
    # land on the pages' disk totals within 3%.
    n = fx["layers"] * (fx["experts_per_layer"] + 1)
    for bits, disk in ((4, fx["disk_gb_4bit"]), (2, fx["disk_gb_2bit"])):
        total_gib = (n * oracle.blob_bytes(H, I, bits)) / 2**30 + fx["non_expert_gb"]
        assert abs(total_gib - disk) / disk < 0.03
    # the generator agrees with the oracle on the layout size
    assert synth.blob_bytes(H, I, 4) == fx["blob_bytes_4bit"]


# ----------------------------------------------------------------------------- hand example


def _hand_blob(spec, H, I, bits):
    def m(d):
        return (d["q"], d["scale"], d["bias"])
    return make_blob(H, I, bits, m(spec["gate"]), m(spec["up"]), m(spec["down"]))


def test_two_expert_hand_example(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "two_expert_example.json")))
    H, I, bits, E, K = fx["hidden"], fx["inter"], fx["bits"], fx["n_experts"], fx["top_k"]
    ex = fx["expected"]
    x = bf16_bits(np.full(H, fx["x_all"], dtype=np.float32))
    wr = bf16_bits(np.repeat(np.array(fx["router_rows_all"], dtype=np.float32)[:, None], H, axis=1))
    blobs = {0: _hand_blob(fx["experts"]["0"], H, I, bits), 1: _hand_blob(fx["experts"]["1"], H, I, bits),
             2: _hand_blob(fx["experts"]["shared"], H, I, bits)}
    r = oracle.layer_forward(x, router_w=wr, router_bias=None, norm_w=None, eps=1e-6, top_k=K, hidden=H, inter=I,
                             bits=bits, blob_of=lambda e: blobs[e])
    np.testing.assert_array_equal(r["logits"], np.array(ex["logits"], dtype=np.float32))
    assert list(r["idx"]) == ex["idx"]
    np.testing.assert_allclose(r["w"], ex["w"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(r["y"][0], ex["y_expert0_all"], rtol=1e-14)
    np.testing.assert_allclose(r["y"][1], ex["y_expert1_all"], rtol=1e-14)
    np.testing.assert_allclose(r["y_shared"], ex["y_shared_all"], rtol=1e-14)
    np.testing.assert_allclose(r["out_f64"], ex["out_f64_all"], rtol=1e-14)
    assert np.all(oracle.bf16_to_f64(r["out"]) == ex["out_bf16_all"])
    # the same numbers from closed forms evaluated here
    w0 = math.exp(1) / (math.exp(1) + math.exp(-1))
    y1 = 64 * 2**-5 * silu(4.0) * 8
    assert abs(r["out_f64"][0] - (1 + w0 * 64 + (1 - w0) * y1 + silu(1.0))) < 1e-12


# ----------------------------------------------------------------------------- dequantisation


@pytest.mark.parametrize("bits", [4, 2])
def test_dequant_identity_every_code(bits):
    """scale 1, bias 0: the dequantised weight is the code itself, for every
    code value, and codes land at the canonical bit positions."""
    H, I = 128, 64
    rng = np.random.default_rng(bits)
    qg = rng.integers(0, 1 << bits, size=(I, H))
    qg[0, :] = np.arange(H) % (1 << bits)
    blob = make_blob(H, I, bits, (qg, 1.0, 0.0), (0, 1.0, 0.0), (0, 1.0, 0.0))
    for r in (0, 1, 17, I - 1):
        for c in range(H):
            assert oracle.weight(blob, H, I, bits, 0, r, c) == qg[r, c]


@pytest.mark.parametrize("bits", [4, 2])
def test_one_hot_input_pins_orientation_and_group(bits):
    """With z = e_c, gate row r equals W[r][c] = s[r][c/64] q[r][c] + b[r][c/64]:
    pins row/column orientation and that the group index is c/64 along the row."""
    H, I = 256, 64
    rng = np.random.default_rng(7)
    q = rng.integers(0, 1 << bits, size=(I, H))
    s = 2.0 ** -rng.integers(0, 6, size=(I, H // 64)).astype(np.float32)
    b = (rng.integers(-8, 8, size=(I, H // 64)) * 2.0**-7).astype(np.float32)
    blob = make_blob(H, I, bits, (q, s, b), (0, 1.0, 0.0), (0, 1.0, 0.0))
    for c in (0, 1, 63, 64, 130, 255):
        z = np.zeros(H, dtype=np.float32)
        z[c] = 1.0
        _, g, _, _ = oracle.expert(blob, H, I, bits, bf16_bits(z))
        want = s[:, c // 64] * q[:, c] + b[:, c // 64]
        np.testing.assert_array_equal(g, want.astype(np.float64))


def test_factored_form_equals_direct_form():
    """sum_g s_g (sum_c q_c z_c) + b_g (sum_c z_c) equals the oracle's direct
    sum_c (s q + b) z_c on random data (the factorisation the kernels use)."""
    wl = synth.WORKLOADS["tiny"]
    H, I = wl.hidden, wl.inter
    blob = synth.expert_blob(wl, 0, 3)
    z = synth.token(wl, 5)
    _, g, _, _ = oracle.expert(blob, H, I, 4, z)
    zf = oracle.bf16_to_f64(z)
    # unpack with numpy from the canonical definition
    words = np.frombuffer(blob[: I * H // 2].tobytes(), dtype="<u4").reshape(I, H // 8)
    q = np.stack([(words >> (4 * j)) & 0xF for j in range(8)], axis=-1).reshape(I, H).astype(np.float64)
    sb = np.frombuffer(blob[I * H // 2: I * H // 2 + 4 * I * (H // 64)].tobytes(), dtype="<u2")
    s = oracle.bf16_to_f64(sb[: I * H // 64]).reshape(I, H // 64)
    b = oracle.bf16_to_f64(sb[I * H // 64:]).reshape(I, H // 64)
    qz = (q * zf).reshape(I, H // 64, 64).sum(-1)
    zs = zf.reshape(H // 64, 64).sum(-1)
    fact = (s * qz + b * zs[None, :]).sum(-1)
    np.testing.assert_allclose(g, fact, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- routing


def test_topk_agrees_with_full_sort():
    rng = np.random.default_rng(0)
    for trial in range(10000):
        E = int(rng.integers(2, 40))
        K = int(rng.integers(1, E + 1))
        logits = rng.standard_normal(E).astype(np.float32)
        if trial % 5 == 0:  # exact ties
            logits[rng.integers(0, E, size=E // 2)] = logits[0]
        idx, w, p = oracle.topk(logits, K)
        order = np.lexsort((np.arange(E), -logits.astype(np.float64)))
        assert list(idx) == list(order[:K])
        assert abs(w.sum() - 1.0) < 1e-12


def test_topk_signed_zeros_tie_by_index():
    """-0 and +0 logits are equal, so they break by the lower index like any tie
    (the reading both sides take; the kernels map -0 to +0 before ranking)."""
    logits = np.array([-1.0, -0.0, 0.0, -0.0, 0.0, -2.0], dtype=np.float32)
    idx, w, _ = oracle.topk(logits, 4)
    assert list(idx) == [1, 2, 3, 4]
    np.testing.assert_allclose(w, [0.25] * 4, rtol=0, atol=1e-15)
    idx, _, _ = oracle.topk(-logits[::-1].copy(), 3)  # [2, -0, 0, -0, 0, 1]: 2, 1, then the lowest-index zero
    assert list(idx) == [0, 5, 1]


def test_topk_weights_full_softmax_when_k_equals_e():
    rng = np.random.default_rng(1)
    logits = (rng.standard_normal(32) * 3).astype(np.float32)
    idx, w, p = oracle.topk(logits, 32)
    l = logits.astype(np.float64)
    sm = np.exp(l - l.max())
    sm /= sm.sum()
    np.testing.assert_allclose(p, sm, rtol=1e-14)
    np.testing.assert_allclose(w, sm[idx], rtol=1e-14)


def test_topk_is_stable_for_huge_logits():
    logits = np.array([1000.0, 999.0, -1000.0, 998.0], dtype=np.float32)
    idx, w, _ = oracle.topk(logits, 2)
    assert list(idx) == [0, 1]
    np.testing.assert_allclose(w, [1 / (1 + math.exp(-1)), 1 / (1 + math.exp(1))], rtol=1e-14)


def test_topk_underflowed_probabilities_rank_by_logit():
    """Probabilities that underflow to 0 in double still rank by their logits:
    selecting the K largest probabilities is selecting the K largest logits."""
    logits = np.array([0.0, -1000.0, -800.0, -900.0, -800.0], dtype=np.float32)
    idx, w, p = oracle.topk(logits, 4)
    assert p[1] == 0.0 and p[2] == 0.0  # exp(-800) underflows
    assert list(idx) == [0, 2, 4, 3]
    np.testing.assert_allclose(w, [1.0, 0.0, 0.0, 0.0], rtol=0, atol=0)


def test_topk_infinite_logits_take_the_softmax_limit():
    """+inf logits share the mass equally (the limit of the softmax as those
    logits grow together); the picks after them rank by logit."""
    inf = np.float32(np.inf)
    logits = np.array([1.0, inf, -3.0, inf, 2.0, inf], dtype=np.float32)
    idx, w, p = oracle.topk(logits, 5)
    assert list(idx) == [1, 3, 5, 4, 0]
    np.testing.assert_allclose(w, [1 / 3, 1 / 3, 1 / 3, 0, 0], rtol=1e-15, atol=0)
    np.testing.assert_allclose(p, [0, 1 / 3, 0, 1 / 3, 0, 1 / 3], rtol=1e-15, atol=0)
    idx, w, _ = oracle.topk(logits, 2)
    assert list(idx) == [1, 3]
    np.testing.assert_allclose(w, [0.5, 0.5], rtol=1e-15, atol=0)


def test_topk_all_minus_inf_or_nan_is_uniform():
    """Every logit -inf (NaN counts as -inf): all experts tie, so the lowest
    indices are picked with equal weights; a single finite logit takes all."""
    logits = np.array([np.nan, -np.inf, np.nan, -np.inf, -np.inf], dtype=np.float32)
    idx, w, p = oracle.topk(logits, 3)
    assert list(idx) == [0, 1, 2]
    np.testing.assert_allclose(w, [1 / 3] * 3, rtol=1e-15, atol=0)
    np.testing.assert_allclose(p, [0.2] * 5, rtol=1e-15, atol=0)
    logits[3] = -7.0
    idx, w, _ = oracle.topk(logits, 3)
    assert list(idx) == [3, 0, 1]
    np.testing.assert_allclose(w, [1.0, 0.0, 0.0], rtol=0, atol=0)


def test_router_bias_shift_and_expert_permutation():
    wl = synth.WORKLOADS["tiny"]
    wr = synth.router_weight(wl, 0)
    z = synth.token(wl, 0)
    rng = np.random.default_rng(3)
    bias = (rng.standard_normal(wl.n_experts) * 0.5).astype(np.float32)
    l0 = oracle.router_logits(wr, bias, z)
    i0, w0, _ = oracle.topk(l0, 4)
    l1 = oracle.router_logits(wr, bias + np.float32(0.25), z)
    i1, w1, _ = oracle.topk(l1, 4)
    assert list(i0) == list(i1)
    np.testing.assert_allclose(w0, w1, atol=1e-6)
    perm = rng.permutation(wl.n_experts)
    l2 = oracle.router_logits(wr[perm], bias[perm], z)
    i2, w2, _ = oracle.topk(l2, 4)
    assert list(perm[i2]) == list(i0)
    np.testing.assert_allclose(w2, w0, rtol=1e-12)


def test_router_logit_is_a_dot_product():
    """One-hot router rows select single input elements."""
    H, E = 128, 8
    z = bf16_bits(np.arange(H, dtype=np.float32) - 60.0)
    wr = np.zeros((E, H), dtype=np.float32)
    for e in range(E):
        wr[e, 10 * e] = 2.0 ** -e
    logits = oracle.router_logits(bf16_bits(wr), None, z)
    np.testing.assert_array_equal(logits, np.array([(10 * e - 60.0) * 2.0**-e for e in range(E)], np.float32))


# ----------------------------------------------------------------------------- expert closed forms


def test_constant_codes_closed_form():
    """Constant codes, scale 1, bias 0: y_j = c_d * I * silu(c_g S) * c_u S with
    S = sum(z)."""
    H, I, bits = 128, 64, 4
    cg, cu, cd = 1, 3, 2
    blob = make_blob(H, I, bits, (cg, 1.0 / 64, 0.0), (cu, 1.0 / 64, 0.0), (cd, 1.0 / 256, 0.0))
    zf = np.full(H, 0.5, dtype=np.float32)
    zf[::3] = -0.25
    S = float(zf.astype(np.float64).sum())
    y, g, u, a = oracle.expert(blob, H, I, bits, bf16_bits(zf))
    gg = cg / 64 * S
    uu = cu / 64 * S
    np.testing.assert_allclose(g, gg, rtol=1e-14)
    np.testing.assert_allclose(u, uu, rtol=1e-14)
    np.testing.assert_allclose(a, silu(gg) * uu, rtol=1e-14)
    np.testing.assert_allclose(y, cd / 256 * I * silu(gg) * uu, rtol=1e-14)


def test_down_projection_orientation():
    """Down codes q[j][i] = j % 16 with scale 1 and constant a: y_j = (j%16) I a."""
    H, I, bits = 128, 64, 4
    qd = np.repeat((np.arange(H) % 16)[:, None], I, axis=1)
    blob = make_blob(H, I, bits, (1, 1.0 / 64, 0.0), (1, 1.0 / 64, 0.0), (qd, 1.0, 0.0))
    z = bf16_bits(np.ones(H, dtype=np.float32))
    y, g, u, a = oracle.expert(blob, H, I, bits, z)
    gg = H / 64.0
    np.testing.assert_allclose(y, (np.arange(H) % 16) * I * silu(gg) * gg, rtol=1e-14)


def test_swiglu_applies_silu_to_gate_not_up():
    H, I, bits = 64, 64, 4
    blob = make_blob(H, I, bits, (1, 1.0 / 16, 0.0), (1, 1.0 / 8, 0.0), (1, 1.0, 0.0))
    y, g, u, a = oracle.expert(blob, H, I, bits, bf16_bits(np.ones(H, dtype=np.float32)))
    assert g[0] == 4.0 and u[0] == 8.0
    np.testing.assert_allclose(a, silu(4.0) * 8.0, rtol=1e-14)
    assert abs(a[0] - silu(8.0) * 4.0) > 0.1


def test_doubling_down_scale_and_bias_doubles_output():
    wl = synth.WORKLOADS["tiny"]
    H, I = wl.hidden, wl.inter
    blob = synth.expert_blob(wl, 0, 1)
    z = synth.token(wl, 2)
    y, *_ = oracle.expert(blob, H, I, 4, z)
    blob2 = blob.copy()
    off = 2 * (I * H // 2 + 4 * I * (H // 64)) + H * I // 2
    n = H * (I // 64)
    sb = np.frombuffer(blob2[off: off + 4 * n].tobytes(), dtype="<u2").copy()
    v = sb.astype(np.uint32)
    exp_field = (v >> 7) & 0xFF
    nz = (v & 0x7FFF) != 0
    assert np.all((exp_field[nz] > 0) & (exp_field[nz] < 254))  # normal, no overflow when doubled
    v[nz] += 1 << 7  # exponent + 1: exact doubling of every non-zero bf16
    blob2[off: off + 4 * n] = np.frombuffer(v.astype("<u2").tobytes(), dtype=np.uint8)
    y2, *_ = oracle.expert(blob2, H, I, 4, z)
    np.testing.assert_array_equal(y2, 2 * y)


# ----------------------------------------------------------------------------- norm and combine


@pytest.mark.parametrize("c", [1.0, 2.0**-10, 3.0, -0.5])
def test_rmsnorm_constant_vector(c):
    H = 256
    h = bf16_bits(np.full(H, c, dtype=np.float32))
    z = oracle.rmsnorm(h, None, 1e-6)
    want = synth.double_to_bf16(c / math.sqrt(c * c + 1e-6))
    assert np.all(z == want)


def test_rmsnorm_uses_mean_and_weight():
    H = 128
    hv = np.where(np.arange(H) % 2 == 0, 2.0, -2.0).astype(np.float32)
    wv = (1.0 + (np.arange(H) % 4) * 0.25).astype(np.float32)
    z = oracle.rmsnorm(bf16_bits(hv), bf16_bits(wv), 1e-6)
    r = 1.0 / math.sqrt(4.0 + 1e-6)
    want = [synth.double_to_bf16(float(hv[i]) * r * float(wv[i])) for i in range(H)]
    assert list(z) == want


def test_combine_is_residual_plus_weighted_sum():
    H, K = 64, 3
    h = bf16_bits(((np.arange(H) - 32) / 8.0).astype(np.float32))
    w = np.array([0.5, 0.25, 0.25])
    ys = np.stack([np.full(H, 1.0), np.full(H, 2.0), np.full(H, -4.0)])
    ysh = np.full(H, 0.125)
    out64, out = oracle.combine(h, w, ys, ysh)
    np.testing.assert_allclose(out64, oracle.bf16_to_f64(h) + 0.5 + 0.5 - 1.0 + 0.125, rtol=1e-14)


def test_round_bf16_ties_to_even():
    assert oracle.round_bf16(1.0 + 2.0**-8) == 0x3F80            # tie -> even (1.0)
    assert oracle.round_bf16(1.0 + 3 * 2.0**-8) == 0x3F82        # tie -> even (1 + 2^-6)
    assert oracle.round_bf16(1.0 + 2.0**-8 + 2.0**-30) == 0x3F81
    assert oracle.round_bf16(-65.59384201648058) == 0xC283        # -65.5
    assert oracle.bf16_value(0x3F81) == 1.0078125


# ---------------------------------------------------------------- 4-bit -> 2-bit requantisation

def _two_bit_grid_blob(H, I, rng):
    """A 2-bit blob whose every group holds codes 0 and 3 (so the group spans the
    whole grid), scale 5 * 2^-6, and an exact bf16 bias per row; and its 4-bit
    expansion q4 = 5 * q2 with scale 2^-6 and the same bias (the same weights)."""
    mats2, mats4 = [], []
    for R, C in ((I, H), (I, H), (H, I)):
        q2 = rng.integers(0, 4, size=(R, C))
        q2[:, 0::64] = 0
        q2[:, 1::64] = 3
        bias = ((np.arange(R) % 5) - 2.0)[:, None] * 2.0 ** -5
        mats2.append((q2, 5 * 2.0 ** -6, bias))
        mats4.append((5 * q2, 2.0 ** -6, bias))
    return make_blob(H, I, 2, *mats2), make_blob(H, I, 4, *mats4)


def test_requant_recovers_an_exact_two_bit_grid():
    rng = np.random.default_rng(3)
    H, I = 256, 128
    b2, b4 = _two_bit_grid_blob(H, I, rng)
    assert np.array_equal(oracle.requant_4to2(b4, H, I), b2)


def test_requant_constant_group_keeps_its_value():
    H, I = 128, 64
    # every weight 7 * 2^-5 + 2^-4 = 0.28125 (exact in bf16)
    b4 = make_blob(H, I, 4, (7, 2.0 ** -5, 2.0 ** -4), (7, 2.0 ** -5, 2.0 ** -4), (7, 2.0 ** -5, 2.0 ** -4))
    out = oracle.requant_4to2(b4, H, I)
    for m, (R, C) in enumerate(((I, H), (I, H), (H, I))):
        for r, c in ((0, 0), (R - 1, C - 1), (R // 2, 65 % C)):
            assert oracle.weight(out, H, I, 2, m, r, c) == 0.28125
    two = make_blob(H, I, 2, (0, 0.0, 0.28125), (0, 0.0, 0.28125), (0, 0.0, 0.28125))
    assert np.array_equal(out, two)


def test_requant_error_bound_and_monotone_codes():
    wl = synth.WORKLOADS["tiny"]
    H, I = wl.hidden, wl.inter
    src = synth.expert_blob(wl, 0, 3)
    out = oracle.requant_4to2(src, H, I)
    assert out.size == oracle.blob_bytes(H, I, 2)
    for m, (R, C) in enumerate(((I, H), (I, H), (H, I))):
        for r in (0, 1, R - 1):
            for g in range(C // 64):
                cols = range(64 * g, 64 * g + 64)
                w4 = np.array([oracle.weight(src, H, I, 4, m, r, c) for c in cols])
                w2 = np.array([oracle.weight(out, H, I, 2, m, r, c) for c in cols])
                lo, hi = w4.min(), w4.max()
                s2 = (w2.max() - w2.min()) / 3 if w2.max() > w2.min() else 0.0
                step = (hi - lo) / 3
                bound = 0.5 * step * (1 + 2.0 ** -7) + 2.0 ** -8 * (abs(lo) + (hi - lo)) + 1e-12
                assert np.max(np.abs(w2 - w4)) <= bound, (m, r, g)
                order = np.argsort(w4, kind="stable")
                assert np.all(np.diff(w2[order]) >= 0), (m, r, g)  # codes follow the weights
                assert s2 <= step * (1 + 2.0 ** -8) + 1e-12


def test_requant_full_shape_size():
    assert oracle.blob_bytes(4096, 1024, 2) == 3_932_160
