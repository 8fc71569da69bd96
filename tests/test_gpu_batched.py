"""The batched (grouped per-expert GEMM) path for T tokens at once, through the
C ABI, against the oracle: same selection, same tolerances as the batch-1 path.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from moe_cases import REL_L2_TOL, W_TOL, Model, OracleLayer, bf16_tensor_bits, rel_l2, tie_free_subseeds

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
TINY2 = dataclasses.replace(TINY, name="tiny2bit", bits=2)
RAGGED = dataclasses.replace(TINY, name="ragged", hidden=320, inter=192, n_experts=37, top_k=3, seed=11)
RAGGED2 = dataclasses.replace(RAGGED, name="ragged2bit", bits=2, seed=12)
ZIPF = dataclasses.replace(TINY, name="tinyzipf", zipf=1.1, seed=14, top_k=4)
STACK = dataclasses.replace(TINY, name="tinystack", n_layers=3, norm=True, seed=13)
WIDE = dataclasses.replace(TINY, name="wide512", n_experts=512, top_k=4, hidden=512, inter=256, seed=15)
SMALL = [TINY, TINY2, RAGGED, RAGGED2, ZIPF, WIDE]


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _flag(name):
    import quantised_expert_ffn_router_b200 as fm
    return getattr(fm, name)


def _tokens(wl, n, layer=0, start=0):
    from synth.gpu import tokens
    idx = list(range(start, start + n))
    return tokens(wl, idx, tie_free_subseeds(wl, layer, idx))


def _check_layer(torch, m, wl, layer, x, T):
    ol = OracleLayer(wl, layer)
    out = torch.empty_like(x)
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    m.fm.fmoe_layer_forward(m.ctx, layer, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), w.data_ptr(), m.stream)
    got = bf16_tensor_bits(out)
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    xb = bf16_tensor_bits(x)
    for t in range(T):
        r = ol.forward(xb[t])
        assert list(gi[t]) == list(r["idx"]), t
        assert np.max(np.abs(gw[t] - r["w"])) <= W_TOL, t
        err = rel_l2(oracle.bf16_to_f64(got[t]), oracle.bf16_to_f64(r["out"]))
        assert err <= REL_L2_TOL, (t, err)
    return out


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_grouped_layer_matches_oracle(torch, wl):
    T = 20
    x = _tokens(wl, T, start=100)
    with Model(wl, flags=_flag("FMOE_FLAG_FORCE_GROUPED")) as m:
        _check_layer(torch, m, wl, 0, x, T)


def test_grouped_layer_spans_several_token_blocks(torch):
    # 70 tokens: the shared expert's segment needs two 64-position work items
    wl = TINY
    T = 70
    x = _tokens(wl, T, start=300)
    with Model(wl) as m:   # default flags: T >= 8 takes the batched path
        _check_layer(torch, m, wl, 0, x, T)


@pytest.mark.parametrize("wl", [TINY, RAGGED2], ids=lambda w: w.name)
def test_grouped_expert_forward_matches_oracle(torch, wl):
    T = 12
    from synth.gpu import tokens
    x = tokens(wl, list(range(500, 500 + T)))
    ol = OracleLayer(wl, 0)
    xb = bf16_tensor_bits(x)
    with Model(wl, flags=_flag("FMOE_FLAG_FORCE_GROUPED")) as m:
        y = torch.empty((T, wl.hidden), dtype=torch.float32, device="cuda")
        for e in [0, wl.n_experts - 1, -1]:
            m.fm.fmoe_expert_forward(m.ctx, 0, e, x.data_ptr(), T, y.data_ptr(), m.stream)
            got = y.cpu().numpy()
            blob = ol.blob(e if e >= 0 else wl.n_experts)
            for t in range(T):
                want, *_ = oracle.expert(blob, wl.hidden, wl.inter, wl.bits, xb[t])
                assert rel_l2(got[t], want) <= REL_L2_TOL, (e, t)


def test_grouped_and_per_token_paths_agree(torch):
    wl = ZIPF
    T = 24
    x = _tokens(wl, T, start=700)
    outs, idxs = [], []
    for flag in ("FMOE_FLAG_FORCE_GROUPED", "FMOE_FLAG_FORCE_PER_TOKEN"):
        with Model(wl, flags=_flag(flag)) as m:
            out = torch.empty_like(x)
            idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
            m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), None, m.stream)
            outs.append(out.float().cpu().numpy())
            idxs.append(idx.cpu().numpy())
    assert np.array_equal(idxs[0], idxs[1])
    for t in range(T):
        assert rel_l2(outs[0][t], outs[1][t]) <= REL_L2_TOL, t


def test_grouped_stack_matches_oracle(torch):
    wl = STACK
    T = 10
    from synth.gpu import tokens
    idx = list(range(T))
    x = tokens(wl, idx, tie_free_subseeds(wl, 0, idx))
    with Model(wl, flags=_flag("FMOE_FLAG_FORCE_GROUPED")) as m:
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
            continue
        assert rel_l2(oracle.bf16_to_f64(got[t]), oracle.bf16_to_f64(h)) <= REL_L2_TOL, t


def test_grouped_path_is_deterministic(torch):
    wl = ZIPF
    T = 32
    x = _tokens(wl, T, start=900)
    with Model(wl) as m:
        a = torch.empty_like(x)
        b = torch.empty_like(x)
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, a.data_ptr(), None, None, m.stream)
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, b.data_ptr(), None, None, m.stream)
        assert torch.equal(a, b)


@pytest.mark.slow
def test_full_batched_step_every_token(torch):
    """The batched workload at full size: 256 tokens per step through the
    grouped path (H 4096, 512 experts with a Zipf(1.1) router skew, top-4 +
    shared, I 1024, 4-bit).  Routing and the layer output are checked for
    every token.  The oracle runs expert by expert (one blob in host memory at
    a time); the routing must give segments of every size class the grouped
    path treats differently (1, 2-15, 16-63 and >= 64 tokens per expert)."""
    wl = synth.WORKLOADS["batched"]
    T, K, E = wl.tokens, wl.top_k, wl.n_experts
    x = _tokens(wl, T)
    with Model(wl) as m:
        out = torch.empty_like(x)
        idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
        w = torch.empty((T, K), dtype=torch.float32, device="cuda")
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), w.data_ptr(), m.stream)
        torch.cuda.synchronize()
        st, word = m.fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == 0, hex(word)
        got, gi, gw = bf16_tensor_bits(out), idx.cpu().numpy(), w.cpu().numpy()
        del m
    torch.cuda.empty_cache()
    ol = OracleLayer(wl, 0)
    xb = bf16_tensor_bits(x)
    ri = np.empty((T, K), np.int64)
    rw = np.empty((T, K))
    for t in range(T):
        i, wt, _ = oracle.topk(oracle.router_logits(ol.router, ol.bias, xb[t]), K)
        ri[t], rw[t] = i, wt
        assert list(gi[t]) == list(i), t
        assert np.max(np.abs(gw[t] - wt)) <= W_TOL, t
    seg = np.bincount(ri.ravel(), minlength=E)
    used = seg[seg > 0]
    for lo, hi in ((1, 1), (2, 15), (16, 63), (64, T)):
        assert np.any((used >= lo) & (used <= hi)), (lo, hi)
    y = np.zeros((T, K, wl.hidden))
    for e in np.unique(ri):  # no norm in this workload: z = x
        blob = synth.expert_blob(wl, 0, int(e))
        for t, k in zip(*np.nonzero(ri == e)):
            y[t, k] = oracle.expert(blob, wl.hidden, wl.inter, wl.bits, xb[t])[0]
    shared = synth.expert_blob(wl, 0, E)
    worst = 0.0
    for t in range(T):
        y_sh = oracle.expert(shared, wl.hidden, wl.inter, wl.bits, xb[t])[0]
        _, want = oracle.combine(xb[t], rw[t], y[t], y_sh)
        err = rel_l2(oracle.bf16_to_f64(got[t]), oracle.bf16_to_f64(want))
        worst = max(worst, err)
        assert err <= REL_L2_TOL, (t, int(seg[ri[t]].min()), err)
