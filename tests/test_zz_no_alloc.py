"""fmoe_route_static -- the router step with its scratch in a fixed device
array, so the call allocates no device memory -- against fmoe_route on the same
inputs.  Two consecutive calls with different tokens check that nothing left in
the fixed scratch by one call leaks into the next.  The file name puts it after
the other GPU tests; it depends on none of their state."""
import dataclasses

import numpy as np
import pytest

import synth
from moe_cases import W_TOL, Model, tie_free_subseeds

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
