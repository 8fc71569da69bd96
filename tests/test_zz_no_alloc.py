"""fmoe_route_static -- the router step with its scratch in a fixed device
array, so the call allocates no device memory -- against the oracle's router
(RMSNorm, logits, softmax, top-K) and against fmoe_route on the same inputs.
Two consecutive calls with different tokens check that nothing left in the
fixed scratch by one call leaks into the next.  That the call allocates
nothing is checked two ways: it is captured into a CUDA graph in global
capture mode (where a cudaMalloc or cudaFree fails the capture) and replayed,
and the device's free memory does not move over many calls.  The file name
puts it after the other GPU tests; it depends on none of their state."""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from moe_cases import W_TOL, Model, bf16_tensor_bits, tie_free_subseeds

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
WIDE = dataclasses.replace(TINY, name="wide512", n_experts=512, top_k=4, seed=21)     # E of the full layer
NORMED = dataclasses.replace(TINY, name="normed", n_layers=2, norm=True, seed=22)     # RMSNorm on the input
ZIPF = dataclasses.replace(TINY, name="zipf", zipf=1.1, top_k=4, seed=23)             # router bias


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _tokens(wl, layer, start, n):
    from synth.gpu import tokens
    idx = list(range(start, start + n))
    return tokens(wl, idx, tie_free_subseeds(wl, layer, idx))


@pytest.mark.parametrize("wl", [TINY, WIDE, NORMED, ZIPF], ids=lambda w: w.name)
def test_static_route_matches_route_on_two_consecutive_calls(torch, wl):
    T, K = 12, wl.top_k
    with Model(wl) as m:
        layer = len(m.weights.layers) - 1
        for call, start in enumerate((0, 40)):
            x = _tokens(wl, layer, start, T)
            idx_a = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
            idx_b = torch.full((T, K), -2, dtype=torch.int32, device="cuda")
            w_a = torch.full((T, K), float("nan"), dtype=torch.float32, device="cuda")
            w_b = torch.full((T, K), float("nan"), dtype=torch.float32, device="cuda")
            m.fm.fmoe_route(m.ctx, layer, x.data_ptr(), T, idx_a.data_ptr(), w_a.data_ptr(), m.stream)
            m.fm.fmoe_route_static(m.ctx, layer, x.data_ptr(), T, idx_b.data_ptr(), w_b.data_ptr(), m.stream)
            torch.cuda.synchronize()
            assert np.array_equal(idx_a.cpu().numpy(), idx_b.cpu().numpy()), (wl.name, call)
            err = float((w_a - w_b).abs().max().item())
            assert err <= W_TOL, (wl.name, call, err)
            assert abs(float(w_b.sum(dim=1).sub(1.0).abs().max().item())) <= 1e-6


def test_static_route_rejects_calls_above_its_scratch(torch):
    import quantised_expert_ffn_router_b200 as fm
    with Model(WIDE) as m:
        T = 32768 // WIDE.n_experts + 1           # one token more than the fixed scratch holds
        x = torch.zeros((T, WIDE.hidden), dtype=torch.bfloat16, device="cuda")
        idx = torch.full((T, WIDE.top_k), -7, dtype=torch.int32, device="cuda")
        w = torch.zeros((T, WIDE.top_k), dtype=torch.float32, device="cuda")
        st = fm.fmoe_route_static(m.ctx, 0, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), m.stream, check=False)
        assert st == fm.FMOE_ERR_UNSUPPORTED
        torch.cuda.synchronize()
        assert bool((idx == -7).all())            # nothing was launched


@pytest.mark.parametrize("wl", [TINY, WIDE, NORMED, ZIPF], ids=lambda w: w.name)
def test_static_route_matches_oracle(torch, wl):
    """Indices bit-exact and weights within 1e-5 of the oracle's router step,
    on the last layer (the normed one for NORMED)."""
    T, K = 12, wl.top_k
    with Model(wl) as m:
        layer = len(m.weights.layers) - 1
        x = _tokens(wl, layer, 100, T)
        idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, K), float("nan"), dtype=torch.float32, device="cuda")
        m.fm.fmoe_route_static(m.ctx, layer, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), m.stream)
        torch.cuda.synchronize()
        gi, gw, xb = idx.cpu().numpy(), w.cpu().numpy(), bf16_tensor_bits(x)
    wr = synth.router_weight(wl, layer)
    bias = synth.zipf_bias(wl, layer)
    norm = synth.norm_weight(wl, layer) if wl.norm else None
    for t in range(T):
        z = oracle.rmsnorm(xb[t], norm, wl.rms_eps) if norm is not None else xb[t]
        want_i, want_w, _ = oracle.topk(oracle.router_logits(wr, bias, z), K)
        assert list(gi[t]) == list(want_i), (wl.name, t)
        assert np.max(np.abs(gw[t] - want_w)) <= W_TOL, (wl.name, t)


def test_static_route_allocates_nothing(torch):
    """Captured in a CUDA graph (global capture mode, so an allocation or free
    inside the call fails the capture) and replayed on new tokens; the free
    device memory is unchanged after 200 eager calls."""
    wl = NORMED
    T, K = 12, wl.top_k
    with Model(wl) as m:
        layer = 1
        x = _tokens(wl, layer, 0, T)
        idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros((T, K), dtype=torch.float32, device="cuda")
        free0 = torch.cuda.mem_get_info()[0]
        for _ in range(200):
            m.fm.fmoe_route_static(m.ctx, layer, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(), m.stream)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
        eager_i, eager_w = idx.clone(), w.clone()

        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side, capture_error_mode="global"):
                st = m.fm.fmoe_route_static(m.ctx, layer, x.data_ptr(), T, idx.data_ptr(), w.data_ptr(),
                                            side.cuda_stream, check=False)
        assert st == m.fm.FMOE_OK, m.fm.fmoe_last_error(m.ctx)
        idx.fill_(-1)
        w.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(idx, eager_i) and torch.equal(w, eager_w)
        x.copy_(_tokens(wl, layer, 40, T))  # new tokens in the captured input buffer
        g.replay()
        m.fm.fmoe_route(m.ctx, layer, x.data_ptr(), T, eager_i.data_ptr(), eager_w.data_ptr(), m.stream)
        torch.cuda.synchronize()
        assert torch.equal(idx, eager_i)
        assert float((w - eager_w).abs().max().item()) <= W_TOL
        del g
