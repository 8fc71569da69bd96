"""4-bit -> 2-bit requantisation (fmoe_requant_4to2) through the C ABI against
the oracle: byte-identical blobs, since both decide codes, scales and biases
with the same fp32 steps."""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from canon import make_blob
from moe_cases import REL_L2_TOL, bf16_tensor_bits, config_for, rel_l2, tie_free_subseeds

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
RAGGED = dataclasses.replace(TINY, name="ragged", hidden=320, inter=192, n_experts=37, top_k=3, seed=11)
LAYER = synth.WORKLOADS["layer"]


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _requant_on_device(torch, src: np.ndarray, n: int, H: int, I: int) -> np.ndarray:
    import quantised_expert_ffn_router_b200 as fm
    d_src = torch.from_numpy(src).cuda()
    d_dst = torch.empty(n * oracle.blob_bytes(H, I, 2), dtype=torch.uint8, device="cuda")
    fm.fmoe_requant_4to2(d_src.data_ptr(), n, H, I, d_dst.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return d_dst.cpu().numpy()


@pytest.mark.parametrize("wl", [TINY, RAGGED, LAYER], ids=lambda w: w.name)
def test_requant_matches_oracle(torch, wl):
    experts = [0, 1, wl.n_experts]  # two routed experts and the shared one
    blobs = [synth.expert_blob(wl, 0, e) for e in experts]
    got = _requant_on_device(torch, np.concatenate(blobs), len(blobs), wl.hidden, wl.inter)
    nb = oracle.blob_bytes(wl.hidden, wl.inter, 2)
    for k, b in enumerate(blobs):
        want = oracle.requant_4to2(b, wl.hidden, wl.inter)
        assert np.array_equal(got[k * nb:(k + 1) * nb], want), experts[k]


def test_requant_recovers_an_exact_two_bit_grid(torch):
    rng = np.random.default_rng(5)
    H, I = 256, 128
    mats2, mats4 = [], []
    for R, C in ((I, H), (I, H), (H, I)):
        q2 = rng.integers(0, 4, size=(R, C))
        q2[:, 0::64] = 0
        q2[:, 1::64] = 3
        bias = ((np.arange(R) % 5) - 2.0)[:, None] * 2.0 ** -5
        mats2.append((q2, 5 * 2.0 ** -6, bias))
        mats4.append((5 * q2, 2.0 ** -6, bias))
    b2, b4 = make_blob(H, I, 2, *mats2), make_blob(H, I, 4, *mats4)
    assert np.array_equal(_requant_on_device(torch, b4, 1, H, I), b2)


def test_requant_rejects_bad_arguments(torch):
    import quantised_expert_ffn_router_b200 as fm
    H, I = 256, 128
    n4, n2 = oracle.blob_bytes(H, I, 4), oracle.blob_bytes(H, I, 2)
    buf = torch.zeros(n4 + n2 + 64, dtype=torch.uint8, device="cuda")
    base = buf.data_ptr()
    with pytest.raises(fm.FmoeError) as err:  # destination inside the source
        fm.fmoe_requant_4to2(base, 1, H, I, base + 256)
    assert err.value.status == fm.FMOE_ERR_INVALID_ARG
    with pytest.raises(fm.FmoeError) as err:
        fm.fmoe_requant_4to2(base + 8, 1, H, I, base + n4 + 16)
    assert err.value.status == fm.FMOE_ERR_ALIGNMENT
    with pytest.raises(fm.FmoeError) as err:
        fm.fmoe_requant_4to2(base, 1, 100, I, base + n4)
    assert err.value.status == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_requant_4to2(base, 0, H, I, base) == fm.FMOE_OK  # nothing to do


def test_requantised_blobs_drive_a_two_bit_layer(torch):
    """Blobs requantised on the device, repacked by fmoe_create for 2 bits, give
    the oracle's 2-bit layer over the oracle's own requantisation."""
    import quantised_expert_ffn_router_b200 as fm
    wl = TINY
    wl2 = dataclasses.replace(wl, bits=2)
    H, I, E = wl.hidden, wl.inter, wl.n_experts
    src = np.concatenate([synth.expert_blob(wl, 0, e) for e in range(E + 1)])
    stream = torch.cuda.current_stream().cuda_stream
    d_src = torch.from_numpy(src).cuda()
    experts = torch.empty((E + 1) * oracle.blob_bytes(H, I, 2), dtype=torch.uint8, device="cuda")
    fm.fmoe_requant_4to2(d_src.data_ptr(), E + 1, H, I, experts.data_ptr(), stream)
    router = torch.from_numpy(synth.router_weight(wl, 0).view(np.int16)).cuda()
    desc = fm.LayerDesc(router_w_dev=router.data_ptr(), router_bias_dev=0, experts_dev=experts.data_ptr(),
                        norm_w_dev=0)
    _, ctx = fm.fmoe_create(config_for(wl2, 1), [desc], stream)
    try:
        idx = list(range(6))
        from synth.gpu import tokens
        x = tokens(wl, idx, tie_free_subseeds(wl, 0, idx))
        out = torch.empty_like(x)
        fm.fmoe_layer_forward(ctx, 0, x.data_ptr(), len(idx), out.data_ptr(), None, None, stream)
        torch.cuda.synchronize()
        got = bf16_tensor_bits(out)
    finally:
        fm.fmoe_destroy(ctx)
    blobs2 = {}

    def blob_of(e):
        if e not in blobs2:
            blobs2[e] = oracle.requant_4to2(synth.expert_blob(wl, 0, e), H, I)
        return blobs2[e]

    xb = bf16_tensor_bits(x)
    rw = synth.router_weight(wl, 0)
    for t in range(len(idx)):
        r = oracle.layer_forward(xb[t], router_w=rw, router_bias=None, norm_w=None, eps=wl.rms_eps, top_k=wl.top_k,
                                 hidden=H, inter=I, bits=2, blob_of=blob_of)
        assert rel_l2(oracle.bf16_to_f64(got[t]), oracle.bf16_to_f64(r["out"])) <= REL_L2_TOL, t
