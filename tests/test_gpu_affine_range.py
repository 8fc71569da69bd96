"""Expert scales and biases far from the synthetic ranges, on both paths.

Both the batch-1 kernel and the grouped path multiply exact integer codes on
the tensor cores and apply the bf16 scale and bias afterwards in fp32
(s * sum(q*x) + b * sum(x) per 64-column group), so no scale or bias ever
passes through fp16.  Scales of 2^-20 (an fp16 subnormal), biases up to 1e5
(above fp16's largest finite value) and scales of 2^-14 with biases to 3e4
must all match the oracle, through the grouped path (T >= 8 with
FMOE_FLAG_FORCE_GROUPED) and the batch-1 kernel (max_tokens = 1, and
FMOE_FLAG_FORCE_PER_TOKEN).
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from moe_cases import REL_L2_TOL, W_TOL, OracleLayer, bf16_tensor_bits, config_for, rel_l2, tie_free_subseeds

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
TINY_SCALE = dataclasses.replace(TINY, name="scale_2^-20", scale_lo=2.0 ** -20, scale_hi=2.0 ** -20, seed=31)
BIG_BIAS = dataclasses.replace(TINY, name="bias_1e5", bias_lo=-1e5, bias_hi=1e5, seed=32)
EDGE = dataclasses.replace(TINY, name="scale_2^-14_bias_3e4", scale_lo=2.0 ** -14, scale_hi=2.0 ** -14,
                           bias_lo=-3e4, bias_hi=3e4, seed=33)
CASES = [TINY_SCALE, BIG_BIAS, EDGE]


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _check_layer_vs_oracle(torch, fm, ctx, wl, T):
    idx_t = list(range(T))
    from synth.gpu import tokens
    x = tokens(wl, idx_t, tie_free_subseeds(wl, 0, idx_t))
    out = torch.empty_like(x)
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    fm.fmoe_layer_forward(ctx, 0, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), w.data_ptr(), stream)
    st, word = fm.fmoe_poll_status(ctx, stream)
    assert st == 0 and word == 0
    got, gi, gw, xb = bf16_tensor_bits(out), idx.cpu().numpy(), w.cpu().numpy(), bf16_tensor_bits(x)
    ol = OracleLayer(wl, 0)
    for t in range(T):
        r = ol.forward(xb[t])
        assert list(gi[t]) == list(r["idx"]), t
        assert np.max(np.abs(gw[t] - r["w"])) <= W_TOL, t
        err = rel_l2(oracle.bf16_to_f64(got[t]), oracle.bf16_to_f64(r["out"]))
        assert err <= REL_L2_TOL, (wl.name, t, err)


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", ["grouped", "max_tokens_1", "force_per_token"])
def test_extreme_scales_and_biases_match_oracle(torch, wl, mode):
    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights
    weights = DeviceWeights(wl)
    flags, max_tokens, T = {"grouped": (fm.FMOE_FLAG_FORCE_GROUPED, 64, 9),
                            "max_tokens_1": (0, 1, 1),
                            "force_per_token": (fm.FMOE_FLAG_FORCE_PER_TOKEN, 64, 3)}[mode]
    descs = [fm.LayerDesc(**d) for d in weights.descs()]
    stream = torch.cuda.current_stream().cuda_stream
    st, ctx = fm.fmoe_create(config_for(wl, len(descs), flags, max_tokens=max_tokens), descs, stream, check=False)
    assert st == fm.FMOE_OK, fm.fmoe_last_error(None)
    try:
        _check_layer_vs_oracle(torch, fm, ctx, wl, T)
    finally:
        fm.fmoe_destroy(ctx)
