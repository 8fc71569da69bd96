"""Top-K with exact ties, on every selection the library has.

The router weights are zeroed and the router bias holds values with many
exact ties (including -0 against +0), so every logit is exactly its expert's
bias.  The selection must then be the first K entries of the experts sorted
by (larger logit, lower index): the fused kernel's route and layer modes, the
grouped path (T >= 8) and the allocation-free router step all have to agree
with that order exactly, and the renormalised weights with the softmax of
the picked logits.  Non-finite biases are included: NaN ranks as -inf, and an
infinite largest logit gives the softmax's limit (equal weights for the picks
equal to it), the rule the oracle takes.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from moe_cases import Model

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
# zipf > 0 gives each layer a router-bias tensor that the tests overwrite
CASES = [
    dataclasses.replace(TINY, name="ties16", n_experts=16, top_k=2, zipf=1.0, seed=31),
    dataclasses.replace(TINY, name="ties37", n_experts=37, top_k=3, zipf=1.0, seed=32),
    dataclasses.replace(TINY, name="ties512", n_experts=512, top_k=4, zipf=1.0, seed=33),
    dataclasses.replace(TINY, name="ties512k8", n_experts=512, top_k=8, zipf=1.0, seed=34),
    # above 512 experts the fused kernel selects in passes over the logits; above
    # 1023 the grouped path is not available and T >= 8 runs token by token
    dataclasses.replace(TINY, name="ties1000", n_experts=1000, top_k=4, zipf=1.0, seed=35),
    dataclasses.replace(TINY, name="ties2048k8", n_experts=2048, top_k=8, zipf=1.0, seed=36),
]


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _patterns(E):
    rng = np.random.default_rng(E)
    yield "all zero", np.zeros(E, np.float32)
    yield "e mod 5", (np.arange(E) % 5).astype(np.float32)
    yield "few levels", rng.integers(0, 4, E).astype(np.float32) * np.float32(0.25)
    signed_zero = np.where(np.arange(E) % 3 == 0, np.float32(-0.0), np.float32(0.0)).astype(np.float32)
    signed_zero[np.arange(E) % 7 == 6] = np.float32(-1.0)
    yield "signed zeros", signed_zero
    top_last = np.full(E, -2.0, np.float32)
    top_last[-3:] = np.float32(1.5)
    yield "ties at the end", top_last
    plus_inf = np.full(E, -1.0, np.float32)
    plus_inf[[1, E // 2, E - 1]] = np.inf
    yield "+inf ties", plus_inf
    yield "all -inf", np.full(E, -np.inf, np.float32)
    nan_mix = np.full(E, np.nan, np.float32)
    nan_mix[::4] = -np.inf
    nan_mix[E // 3] = np.float32(0.5)
    yield "NaN and -inf", nan_mix


def _expected(bias, K):
    """Order (larger logit, lower index; NaN as -inf) and renormalised weights;
    an infinite largest logit gives the softmax's limit, equal shares for the
    picks equal to it."""
    lg = np.where(np.isnan(bias), -np.inf, bias).astype(np.float64)
    order = sorted(range(len(lg)), key=lambda e: (-lg[e], e))[:K]
    logits = lg[order]
    if np.isinf(logits[0]):
        w = (logits == logits[0]).astype(np.float64)
    else:
        w = np.exp(logits - logits[0])
    return np.array(order, np.int32), w / w.sum()


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_topk_exact_ties(torch, wl):
    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import tokens
    E, K = wl.n_experts, wl.top_k
    T = 8  # the grouped path takes T >= 8
    x = tokens(wl, range(T))
    with Model(wl) as m:
        layer = m.weights.layers[0]
        layer.router.zero_()
        for name, bias in _patterns(E):
            layer.bias.copy_(torch.from_numpy(bias))
            want_idx, want_w = _expected(bias, K)
            o_idx, o_w, _ = oracle.topk(bias, K)  # the oracle takes the same rule
            assert np.array_equal(o_idx, want_idx) and np.allclose(o_w, want_w, rtol=0, atol=1e-15), name
            got = {}
            idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
            w = torch.empty((T, K), dtype=torch.float32, device="cuda")
            m.fm.fmoe_route(m.ctx, 0, x[:1].data_ptr(), 1, idx.data_ptr(), w.data_ptr(), m.stream)
            got["route"] = (idx[:1].clone(), w[:1].clone())
            out = torch.empty_like(x)
            m.fm.fmoe_layer_forward(m.ctx, 0, x[:1].data_ptr(), 1, out.data_ptr(), idx.data_ptr(), w.data_ptr(),
                                    m.stream)
            got["layer"] = (idx[:1].clone(), w[:1].clone())
            m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), w.data_ptr(),
                                    m.stream)
            got["grouped"] = (idx.clone(), w.clone())
            m.fm.fmoe_route_static(m.ctx, 0, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), m.stream)
            got["static"] = (idx.clone(), w.clone())
            st, word = fm.fmoe_poll_status(m.ctx, m.stream)
            assert st == 0, hex(word)
            for path, (gi, gw) in got.items():
                gi, gw = gi.cpu().numpy(), gw.cpu().numpy()
                for t in range(gi.shape[0]):
                    assert np.array_equal(gi[t], want_idx), (name, path, t, gi[t], want_idx)
                    assert np.allclose(gw[t], want_w, rtol=0, atol=1e-6), (name, path, t, gw[t], want_w)
