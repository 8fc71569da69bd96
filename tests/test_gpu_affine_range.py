"""Expert scales and biases at the edges of what the kernels represent exactly.

The batch-1 kernel applies the bf16 scale and bias in fp32 (s * sum(q*x) +
b * sum(x)), so any finite bf16 value is exact there.  The grouped path
dequantises w = q*s + b in fp16 on fp16 copies of s and b, which needs the
scale to be 0 or of magnitude in [2^-14, 65504], the bias at most 65504 in
magnitude and no |w| above 65504.  A context that may take the grouped path
must refuse other weights at create, before it rewrites them; one that never
does (max_tokens = 1, or FMOE_FLAG_FORCE_PER_TOKEN) must accept them and
match the oracle.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from moe_cases import REL_L2_TOL, W_TOL, OracleLayer, bf16_tensor_bits, config_for, rel_l2, tie_free_subseeds

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
# scales of 2^-20: an fp16 subnormal
TINY_SCALE = dataclasses.replace(TINY, name="scale_2^-20", scale_lo=2.0 ** -20, scale_hi=2.0 ** -20, seed=31)
# biases up to 1e5: above fp16's largest finite value
BIG_BIAS = dataclasses.replace(TINY, name="bias_1e5", bias_lo=-1e5, bias_hi=1e5, seed=32)
# the smallest accepted scale and biases up to 3e4: inside the grouped path's range
EDGE = dataclasses.replace(TINY, name="fp16_edge", scale_lo=2.0 ** -14, scale_hi=2.0 ** -14, bias_lo=-3e4,
                           bias_hi=3e4, seed=33)


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _create(torch, wl, weights, flags, max_tokens):
    import quantised_expert_ffn_router_b200 as fm
    descs = [fm.LayerDesc(**d) for d in weights.descs()]
    stream = torch.cuda.current_stream().cuda_stream
    return fm.fmoe_create(config_for(wl, len(descs), flags, max_tokens=max_tokens), descs, stream, check=False)


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


@pytest.mark.parametrize("wl,what", [(TINY_SCALE, "scale"), (BIG_BIAS, "bias")], ids=lambda v: getattr(v, "name", v))
def test_grouped_context_rejects_out_of_range_weights_untouched(torch, wl, what):
    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights
    weights = DeviceWeights(wl)
    before = [l.experts.clone() for l in weights.layers]
    for flags in (0, fm.FMOE_FLAG_FORCE_GROUPED):
        st, ctx = _create(torch, wl, weights, flags, 64)
        assert st == fm.FMOE_ERR_UNSUPPORTED and ctx is None, st
        assert what in fm.fmoe_last_error(None)
        torch.cuda.synchronize()
        for a, layer in zip(before, weights.layers):
            assert torch.equal(a, layer.experts)  # still the canonical blobs


@pytest.mark.parametrize("wl", [TINY_SCALE, BIG_BIAS], ids=lambda w: w.name)
@pytest.mark.parametrize("mode", ["max_tokens_1", "force_per_token"])
def test_batch1_kernel_takes_out_of_range_weights(torch, wl, mode):
    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights
    weights = DeviceWeights(wl)
    flags, max_tokens = (0, 1) if mode == "max_tokens_1" else (fm.FMOE_FLAG_FORCE_PER_TOKEN, 64)
    st, ctx = _create(torch, wl, weights, flags, max_tokens)
    assert st == fm.FMOE_OK, fm.fmoe_last_error(None)
    try:
        _check_layer_vs_oracle(torch, fm, ctx, wl, 1 if max_tokens == 1 else 3)
    finally:
        fm.fmoe_destroy(ctx)


def test_grouped_path_at_the_edge_of_its_range(torch):
    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights
    wl = EDGE
    weights = DeviceWeights(wl)
    st, ctx = _create(torch, wl, weights, fm.FMOE_FLAG_FORCE_GROUPED, 64)
    assert st == fm.FMOE_OK, fm.fmoe_last_error(None)
    try:
        _check_layer_vs_oracle(torch, fm, ctx, wl, 9)
    finally:
        fm.fmoe_destroy(ctx)
