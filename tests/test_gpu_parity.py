"""CUDA path vs the CPU oracle, through the C ABI, on seeded synthetic inputs.

Index work (packed layout round trip, top-K indices) must be bit-exact; the
router weights agree to 1e-5 absolute; expert and layer outputs to a per-token
relative L2 error of 2e-3 (bf16 I/O, fp32 accumulation).  Inputs are redrawn
until the oracle's top-(K+1) logits are separated by at least 1e-3, so the
selection is unique and both sides must find it.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from moe_cases import (REL_L2_TOL, W_TOL, Model, OracleLayer, bf16_tensor_bits, rel_l2, tie_free_subseeds)

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
TINY2 = dataclasses.replace(TINY, name="tiny2bit", bits=2)
# ragged: hidden and inter not multiples of 256, odd expert count
RAGGED = dataclasses.replace(TINY, name="ragged", hidden=320, inter=192, n_experts=37, top_k=3, seed=11)
RAGGED2 = dataclasses.replace(RAGGED, name="ragged2bit", bits=2, seed=12)
STACK = dataclasses.replace(TINY, name="tinystack", n_layers=3, norm=True, seed=13)
ZIPF = dataclasses.replace(TINY, name="tinyzipf", zipf=1.1, seed=14, top_k=4)
LAYER = synth.WORKLOADS["layer"]
SMALL = [TINY, TINY2, RAGGED, RAGGED2, ZIPF]


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _tokens(wl, n, layer=0, start=0):
    idx = list(range(start, start + n))
    sub = tie_free_subseeds(wl, layer, idx)
    from synth.gpu import tokens
    return idx, sub, tokens(wl, idx, sub)


def test_device_tokens_match_host_generator(torch):
    # a contiguous range is drawn by one launch; it must give the host bytes
    from synth.gpu import tokens
    for wl in (TINY, LAYER):
        got = tokens(wl, range(5, 12)).view(torch.int16).cpu().numpy().view(np.uint16)
        for r, t in enumerate(range(5, 12)):
            assert np.array_equal(got[r], synth.token(wl, t)), (wl.name, t)


@pytest.mark.parametrize("wl", SMALL + [STACK], ids=lambda w: w.name)
def test_packed_layout_round_trip(torch, wl):
    with Model(wl) as m:
        blob = wl.blob_bytes
        dst = torch.empty(blob, dtype=torch.uint8, device="cuda")
        for layer in range(len(m.weights.layers)):
            want = synth.expert_blobs(wl, layer, 0, wl.n_experts + 1)
            for e in list(range(wl.n_experts)) + [-1]:
                m.fm.fmoe_unpack_expert(m.ctx, layer, e, dst.data_ptr(), m.stream)
                got = dst.cpu().numpy()
                assert np.array_equal(got, want[e if e >= 0 else wl.n_experts]), (layer, e)


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_route_matches_oracle(torch, wl):
    T = 8
    _, sub, x = _tokens(wl, T)
    ol = OracleLayer(wl, 0)
    with Model(wl) as m:
        idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
        m.fm.fmoe_route(m.ctx, 0, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), m.stream)
        idx, w = idx.cpu().numpy(), w.cpu().numpy()
    xb = bf16_tensor_bits(x)
    for t in range(T):
        z = oracle.rmsnorm(xb[t], ol.norm, wl.rms_eps) if ol.norm is not None else xb[t]
        oi, ow, _ = oracle.topk(oracle.router_logits(ol.router, ol.bias, z), wl.top_k)
        assert list(idx[t]) == list(oi), t
        assert np.max(np.abs(w[t] - ow)) <= W_TOL, t


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_expert_forward_matches_oracle(torch, wl):
    T = 3
    _, sub, x = _tokens(wl, T, start=20)
    ol = OracleLayer(wl, 0)
    xb = bf16_tensor_bits(x)
    experts = sorted(set([0, 1, wl.n_experts - 1, wl.n_experts // 2])) + [-1]
    with Model(wl) as m:
        y = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
        for e in experts:
            m.fm.fmoe_expert_forward(m.ctx, 0, e, x.data_ptr(), T, y.data_ptr(), m.stream)
            got = y.cpu().numpy()
            blob = ol.blob(e if e >= 0 else wl.n_experts)
            for t in range(T):
                want, *_ = oracle.expert(blob, wl.hidden, wl.inter, wl.bits, xb[t])
                err = rel_l2(got[t], want)
                assert err <= REL_L2_TOL, (e, t, err)


def _check_layer(torch, m, wl, layer, x, T):
    ol = OracleLayer(wl, layer)
    out = torch.empty_like(x)
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    m.fm.fmoe_layer_forward(m.ctx, layer, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), w.data_ptr(), m.stream)
    got = bf16_tensor_bits(out)
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    xb = bf16_tensor_bits(x)
    worst = 0.0
    for t in range(T):
        r = ol.forward(xb[t])
        assert list(gi[t]) == list(r["idx"]), t
        assert np.max(np.abs(gw[t] - r["w"])) <= W_TOL, t
        err = rel_l2(oracle.bf16_to_f64(got[t]), oracle.bf16_to_f64(r["out"]))
        worst = max(worst, err)
        assert err <= REL_L2_TOL, (t, err)
    return worst


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_layer_forward_matches_oracle(torch, wl):
    T = 6
    _, _, x = _tokens(wl, T, start=40)
    with Model(wl) as m:
        _check_layer(torch, m, wl, 0, x, T)


# more experts than one lane-per-16-entries pass covers (the fused kernel's
# top-K then runs in passes); 2048 is above the grouped path's limit, so T >= 8
# runs token by token there
MANY_E = [dataclasses.replace(TINY, name="experts1000", n_experts=1000, top_k=4, seed=15),
          dataclasses.replace(TINY, name="experts2048k8", n_experts=2048, top_k=8, seed=16)]


@pytest.mark.parametrize("wl", MANY_E, ids=lambda w: w.name)
def test_many_experts_match_oracle(torch, wl):
    for T in (3, 8):
        _, _, x = _tokens(wl, T, start=80)
        with Model(wl) as m:
            _check_layer(torch, m, wl, 0, x, T)
            idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
            w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
            m.fm.fmoe_route(m.ctx, 0, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), m.stream)
            st, word = m.fm.fmoe_poll_status(m.ctx, m.stream)
            assert st == 0, hex(word)
            gi, gw = idx.cpu().numpy(), w.cpu().numpy()
        ol = OracleLayer(wl, 0)
        xb = bf16_tensor_bits(x)
        for t in range(T):
            r = ol.forward(xb[t])
            assert list(gi[t]) == list(r["idx"]), (T, t)
            assert np.max(np.abs(gw[t] - r["w"])) <= W_TOL, (T, t)


def test_layer_equals_sum_of_route_and_experts(torch):
    """layer(h) = bf16(h + y_shared + sum_k w_k y_k) using the library's own
    route and expert calls (fp32, same accumulation order)."""
    wl = TINY
    T = 4
    _, _, x = _tokens(wl, T, start=60)
    with Model(wl) as m:
        out = torch.empty_like(x)
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, out.data_ptr(), None, None, m.stream)
        idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
        m.fm.fmoe_route(m.ctx, 0, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), m.stream)
        y = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
        acc = x.float().clone()
        m.fm.fmoe_expert_forward(m.ctx, 0, -1, x.data_ptr(), T, y.data_ptr(), m.stream)
        acc += y
        for t in range(T):
            for k in range(wl.top_k):
                m.fm.fmoe_expert_forward(m.ctx, 0, int(idx[t, k]), x[t:t + 1].data_ptr(), 1, y.data_ptr(), m.stream)
                acc[t] = torch.addcmul(acc[t], w[t, k], y[0])
        ref = acc.to(torch.bfloat16)
        assert rel_l2(out.float().cpu().numpy(), ref.float().cpu().numpy()) < 1e-3


def test_stack_matches_oracle(torch):
    wl = STACK
    T = 4
    idx = list(range(T))
    from synth.gpu import tokens
    # the first layer's routing must be tie-free; deeper layers are checked for
    # their oracle margin and reported
    sub = tie_free_subseeds(wl, 0, idx)
    x = tokens(wl, idx, sub)
    with Model(wl) as m:
        out = torch.empty_like(x)
        m.fm.fmoe_stack_forward(m.ctx, 0, wl.n_layers, x.data_ptr(), T, out.data_ptr(), m.stream)
        got = bf16_tensor_bits(out)
    layers = [OracleLayer(wl, l) for l in range(wl.n_layers)]
    xb = bf16_tensor_bits(x)
    for t in range(T):
        h = xb[t]
        margin = np.inf
        for ol in layers:
            r = ol.forward(h)
            margin = min(margin, oracle.topk_gaps(r["logits"], wl.top_k))
            h = r["out"]
        if margin < 1e-4:
            continue  # a near-tie inside the stack: selection not unique
        assert rel_l2(oracle.bf16_to_f64(got[t]), oracle.bf16_to_f64(h)) <= REL_L2_TOL, t


@pytest.mark.slow
def test_full_layer_sampled_tokens(torch):
    """Full shape (H 4096, 512 experts, top-4 + shared, I 1024, 4-bit) at the
    benchmark's launch configuration; the oracle checks sampled tokens."""
    wl = LAYER
    rng = np.random.default_rng(0)
    idx = sorted(rng.choice(wl.tokens, size=8, replace=False).tolist())
    sub = tie_free_subseeds(wl, 0, idx)
    from synth.gpu import tokens
    x = tokens(wl, idx, sub)
    with Model(wl) as m:
        worst = _check_layer(torch, m, wl, 0, x, len(idx))
    assert worst <= REL_L2_TOL


def _full_stack_teacher_forced(torch, wl, idx):
    """Full-size stack, a few tokens.  fmoe_stack_forward must equal the same
    layers chained through fmoe_layer_forward bit for bit, and every layer must
    match the oracle applied to the GPU's own input of that layer (teacher
    forcing; errors of earlier layers are not carried into later checks).
    Layers whose oracle routing has a near-tie are not compared."""
    from synth.gpu import tokens
    T = len(idx)
    x = tokens(wl, idx, tie_free_subseeds(wl, 0, idx))
    with Model(wl) as m:
        out = torch.empty_like(x)
        m.fm.fmoe_stack_forward(m.ctx, 0, wl.n_layers, x.data_ptr(), T, out.data_ptr(), m.stream)
        hs = [x]
        for layer in range(wl.n_layers):
            h = torch.empty_like(x)
            m.fm.fmoe_layer_forward(m.ctx, layer, hs[-1].data_ptr(), T, h.data_ptr(), None, None, m.stream)
            hs.append(h)
        torch.cuda.synchronize()
        st, word = m.fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == 0, hex(word)
        got = [bf16_tensor_bits(h) for h in hs]
        assert np.array_equal(bf16_tensor_bits(out), got[-1])
        del m
    torch.cuda.empty_cache()
    checked = 0
    for layer in range(wl.n_layers):
        ol = OracleLayer(wl, layer)
        for t in range(T):
            r = ol.forward(got[layer][t])
            if oracle.topk_gaps(r["logits"], wl.top_k) < 1e-4:
                continue  # near-tie: the selection is not unique at this precision
            err = rel_l2(oracle.bf16_to_f64(got[layer + 1][t]), oracle.bf16_to_f64(r["out"]))
            assert err <= REL_L2_TOL, (layer, t, err)
            checked += 1
    assert checked >= wl.n_layers  # most (layer, token) pairs are compared


@pytest.mark.slow
def test_full_stack_4bit_teacher_forced(torch):
    """24 layers x (H 4096, 512 experts, top-4 + shared, I 1024, 4-bit) with
    RMSNorm between layers (about 87 GB resident), two tokens."""
    _full_stack_teacher_forced(torch, synth.WORKLOADS["stack4"], [5, 9])


@pytest.mark.slow
def test_full_stack_2bit_teacher_forced(torch):
    """60 layers of the same shape at 2 bits (about 116 GB resident), two tokens."""
    _full_stack_teacher_forced(torch, synth.WORKLOADS["stack2"], [5, 9])


def test_overlapping_buffers_are_rejected(torch):
    """h_out must not overlap h_in: rejected before any GPU work, for the layer
    and the stack call, whole or partial overlap."""
    wl = TINY
    with Model(wl) as m:
        x = torch.zeros((4, wl.hidden), dtype=torch.bfloat16, device="cuda")
        calls = [lambda: m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), 2, x.data_ptr(), None, None, m.stream),
                 lambda: m.fm.fmoe_layer_forward(m.ctx, 0, x[0].data_ptr(), 2, x[1].data_ptr(), None, None, m.stream),
                 lambda: m.fm.fmoe_stack_forward(m.ctx, 0, 1, x[0].data_ptr(), 2, x[1].data_ptr(), m.stream)]
        for call in calls:
            with pytest.raises(m.fm.FmoeError) as err:
                call()
            assert err.value.status == m.fm.FMOE_ERR_INVALID_ARG
            assert "overlaps" in str(err.value)
        m.fm.fmoe_layer_forward(m.ctx, 0, x[0].data_ptr(), 2, x[2].data_ptr(), None, None, m.stream)  # disjoint: fine


def test_deterministic(torch):
    wl = RAGGED
    T = 3
    _, _, x = _tokens(wl, T, start=80)
    with Model(wl) as m:
        a = torch.empty_like(x)
        b = torch.empty_like(x)
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, a.data_ptr(), None, None, m.stream)
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, b.data_ptr(), None, None, m.stream)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_zero_tokens_is_a_no_op(torch):
    wl = TINY
    with Model(wl) as m:
        x = torch.zeros((1, wl.hidden), dtype=torch.bfloat16, device="cuda")
        out = torch.full_like(x, 3.0)
        assert m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), 0, out.data_ptr(), None, None, m.stream) == 0
        torch.cuda.synchronize()
        assert torch.all(out == 3.0)


def test_bounded_wait_reports_timeout(torch):
    """Fault injection on the device without a fault: the router never
    publishes, every block's wait runs out after 20 ms, the status word says
    so, and the context (and a fresh one) stay usable."""
    import quantised_expert_ffn_router_b200 as fm
    wl = TINY
    _, _, x = _tokens(wl, 1, start=90)
    with Model(wl, flags=fm.FMOE_FLAG_DEBUG_SKIP_ROUTER_RELEASE, timeout_us=20000) as m:
        out = torch.empty_like(x)
        fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), 1, out.data_ptr(), None, None, m.stream)
        st, word = fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == fm.FMOE_ERR_TIMEOUT and word != 0
        st, word = fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == fm.FMOE_OK and word == 0
    with Model(wl) as m:
        _check_layer(torch, m, wl, 0, x, 1)
        st, word = fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == fm.FMOE_OK and word == 0
