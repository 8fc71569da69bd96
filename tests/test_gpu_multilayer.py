"""One launch per token through every layer of a stack (the multi-layer
decode kernel behind fmoe_stack_forward) against the per-layer launches.

The multi-layer launch does the same arithmetic in the same order as one
launch per layer, so its output must equal the per-layer path bit for bit:
chained fmoe_layer_forward calls, and fmoe_stack_forward on a context made
with FMOE_FLAG_STACK_PER_LAYER.  The per-layer path itself is checked against
the oracle in test_gpu_parity.py; here the oracle checks the last layer of one
case directly as well.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from moe_cases import REL_L2_TOL, W_TOL, Model, OracleLayer, bf16_tensor_bits, rel_l2, tie_free_subseeds

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
STACK7 = dataclasses.replace(TINY, name="stack7", n_layers=7, norm=True, seed=21)
STACK7_2 = dataclasses.replace(STACK7, name="stack7_2bit", bits=2, seed=22)
RAGGED5 = dataclasses.replace(TINY, name="ragged5", hidden=320, inter=192, n_experts=37, top_k=3, n_layers=5,
                              norm=True, seed=23)
NONORM4 = dataclasses.replace(TINY, name="nonorm4", n_layers=4, norm=False, zipf=1.1, top_k=4, seed=24)
DEEP40 = dataclasses.replace(TINY, name="deep40", n_layers=40, norm=True, seed=25)
CASES = [STACK7, STACK7_2, RAGGED5, NONORM4]


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _x(wl, n, start=0):
    from synth.gpu import tokens
    idx = list(range(start, start + n))
    return tokens(wl, idx, tie_free_subseeds(wl, 0, idx))


def _ok(m):
    st, word = m.fm.fmoe_poll_status(m.ctx, m.stream)
    assert st == 0 and word == 0, hex(word)


def _stack(torch, m, x, lb, le):
    out = torch.empty_like(x)
    m.fm.fmoe_stack_forward(m.ctx, lb, le, x.data_ptr(), x.shape[0], out.data_ptr(), m.stream)
    return out


def _chained(torch, m, x, lb, le):
    h = x
    for layer in range(lb, le):
        nxt = torch.empty_like(x)
        m.fm.fmoe_layer_forward(m.ctx, layer, h.data_ptr(), x.shape[0], nxt.data_ptr(), None, None, m.stream)
        h = nxt
    return h


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_multi_layer_equals_per_layer(torch, wl):
    import quantised_expert_ffn_router_b200 as fm
    x = _x(wl, 3)
    ranges = [(0, wl.n_layers), (1, wl.n_layers - 1)]
    with Model(wl) as m:
        multi = [_stack(torch, m, x, lb, le) for lb, le in ranges]
        chained = [_chained(torch, m, x, lb, le) for lb, le in ranges]
        _ok(m)
        multi = [bf16_tensor_bits(t) for t in multi]
        chained = [bf16_tensor_bits(t) for t in chained]
    for a, b in zip(multi, chained):
        assert np.array_equal(a, b)
    with Model(wl, flags=fm.FMOE_FLAG_STACK_PER_LAYER) as m:
        per_layer = bf16_tensor_bits(_stack(torch, m, x, 0, wl.n_layers))
        _ok(m)
    assert np.array_equal(per_layer, multi[0])


def test_multi_layer_last_layer_matches_oracle(torch):
    """The last layer of a 7-layer launch against the oracle applied to the
    GPU's own input of that layer (the output of a 6-layer launch)."""
    wl = STACK7
    x = _x(wl, 2, start=40)
    with Model(wl) as m:
        h6 = bf16_tensor_bits(_stack(torch, m, x, 0, 6))
        h7 = bf16_tensor_bits(_stack(torch, m, x, 0, 7))
        _ok(m)
    ol = OracleLayer(wl, 6)
    checked = 0
    for t in range(2):
        r = ol.forward(h6[t])
        if oracle.topk_gaps(r["logits"], wl.top_k) < 1e-4:
            continue  # near-tie: the selection is not unique at this precision
        assert rel_l2(oracle.bf16_to_f64(h7[t]), oracle.bf16_to_f64(r["out"])) <= REL_L2_TOL
        checked += 1
    assert checked >= 1


def test_multi_layer_deep_stack_and_interleaving(torch):
    """Forty layers in one launch (every ring stage and down stage changes
    phase many times), and multi-layer and single-layer launches interleaved
    on one context: the per-launch tags stay consistent."""
    wl = DEEP40
    x = _x(wl, 2, start=7)
    with Model(wl) as m:
        full = bf16_tensor_bits(_stack(torch, m, x, 0, 40))
        full_chained = bf16_tensor_bits(_chained(torch, m, x, 0, 40))
        again = bf16_tensor_bits(_stack(torch, m, x, 0, 40))
        mid = _stack(torch, m, x, 3, 17)
        mid_chained = _chained(torch, m, x, 3, 17)
        tail = bf16_tensor_bits(_stack(torch, m, mid, 17, 40))
        tail_chained = bf16_tensor_bits(_chained(torch, m, mid, 17, 40))
        _ok(m)
        mid, mid_chained = bf16_tensor_bits(mid), bf16_tensor_bits(mid_chained)
    assert np.array_equal(full, full_chained)
    assert np.array_equal(full, again)
    assert np.array_equal(mid, mid_chained)
    assert np.array_equal(tail, tail_chained)


def test_multi_layer_bounded_wait_reports_timeout(torch):
    """The router never publishes: the first layer's waits run out after 20 ms,
    the later layers are skipped, the status word says so and a fresh context
    works."""
    import quantised_expert_ffn_router_b200 as fm
    wl = STACK7
    x = _x(wl, 1, start=90)
    with Model(wl, flags=fm.FMOE_FLAG_DEBUG_SKIP_ROUTER_RELEASE, timeout_us=20000) as m:
        _stack(torch, m, x, 0, wl.n_layers)
        st, word = fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == fm.FMOE_ERR_TIMEOUT and word != 0
        st, word = fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == fm.FMOE_OK and word == 0
    with Model(wl) as m:
        a = bf16_tensor_bits(_stack(torch, m, x, 0, wl.n_layers))
        b = bf16_tensor_bits(_chained(torch, m, x, 0, wl.n_layers))
        _ok(m)
    assert np.array_equal(a, b)


def test_tags_survive_the_wrap_past_two_to_the_32(torch):
    """A launch tags its cross-block words epoch + 1 .. epoch + layers.  With
    the epoch set just below 2^32, single- and multi-layer launches run across
    the point where the host clears the tagged words and restarts the count:
    the outputs equal those of a fresh context bit for bit, and the
    single-layer results (indices, weights, output) match the oracle."""
    wl = STACK7
    T = 2  # below the grouped path's threshold: one launch per token
    x = _x(wl, T, start=40)

    def run(m):
        out = torch.empty_like(x)
        idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), w.data_ptr(), m.stream)
        stack = _stack(torch, m, x, 0, wl.n_layers)
        return (bf16_tensor_bits(out), idx.cpu().numpy(), w.cpu().numpy(), bf16_tensor_bits(stack))

    with Model(wl) as m:
        fresh = run(m)
        _ok(m)
    top = 0xFFFFFFFF
    with Model(wl) as m:
        # per run(): 2 single-layer launches (1 tag each), then 2 stack launches (7 tags each)
        for epoch in (top - 20, top - 9, top - 2, top - 1, top):
            m.fm.fmoe_debug_set_epoch(m.ctx, epoch, m.stream)
            for _ in range(2):
                got = run(m)
                _ok(m)
                for a, b in zip(got, fresh):
                    assert np.array_equal(a, b), hex(epoch)
    ol = OracleLayer(wl, 0)
    xb = bf16_tensor_bits(x)
    out, gi, gw, _ = fresh
    for t in range(T):
        r = ol.forward(xb[t])
        assert list(gi[t]) == list(r["idx"]), t
        assert np.max(np.abs(gw[t] - r["w"])) <= W_TOL, t
        assert rel_l2(oracle.bf16_to_f64(out[t]), oracle.bf16_to_f64(r["out"])) <= REL_L2_TOL, t
