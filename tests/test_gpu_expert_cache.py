"""Host-resident routed experts behind the HBM expert cache (fmoe_create_cached).

A cached context reads every byte a resident context reads, only from its
cache slot or from host memory, so its outputs, indices and weights must
equal the resident context's bit for bit, whatever mix of hits, misses and
evictions the cache sees.  The hit and miss counts must equal those of a
host model of the documented CLOCK policy fed with the same routing: that
checks the kernel's bookkeeping (the fill of a miss is checked by every later
hit on that slot, whose output must still be exact).
"""
import dataclasses

import numpy as np
import pytest

import synth
from moe_cases import Model, bf16_tensor_bits, config_for, tie_free_subseeds

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
RAGGED = dataclasses.replace(TINY, name="ragged", hidden=320, inter=192, n_experts=37, top_k=3, seed=41)
TINY2 = dataclasses.replace(TINY, name="tiny2bit", bits=2, seed=42)
ZIPF = dataclasses.replace(TINY, name="zipf", n_experts=64, top_k=4, zipf=1.1, seed=43)
STACK5 = dataclasses.replace(TINY, name="stack5", n_layers=5, norm=True, seed=44)
WINDOW = 32  # slots from the hand a launch may sweep


@pytest.fixture(scope="module")
def torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


class ClockModel:
    """The cache policy as documented: keys layer*E + expert, CLOCK over n slots."""

    def __init__(self, n):
        self.n, self.hand = n, 0
        self.owner, self.ref, self.slot_of = [-1] * n, [0] * n, {}
        self.hits = self.misses = 0

    def step(self, key0, picks):
        n, K = self.n, len(picks)
        have = [self.slot_of.get(key0 + e, -1) for e in picks]
        hit = [h >= 0 for h in have]
        win = [(self.hand + i) % n for i in range(min(WINDOW, n))]
        held = {have[k] for k in range(K) if hit[k]}
        order = [i for i, s in enumerate(win) if s not in held and self.ref[s] == 0]
        order += [i for i, s in enumerate(win) if s not in held and self.ref[s] != 0]
        vpos, r = {}, 0
        for k in range(K):
            if not hit[k]:
                vpos[k] = order[r]
                r += 1
        walk = max(vpos.values()) + 1 if vpos else 0
        cslot = [have[k] if hit[k] else win[vpos[k]] for k in range(K)]
        for w in range(walk):
            s = (self.hand + w) % n
            if s not in cslot:
                self.ref[s] = 0
        for k in range(K):
            v = cslot[k]
            if hit[k]:
                self.hits += 1
            else:
                old = self.owner[v]
                if old >= 0:
                    del self.slot_of[old]
                self.owner[v] = key0 + picks[k]
                self.slot_of[key0 + picks[k]] = v
                self.misses += 1
            self.ref[v] = 1
        self.hand = (self.hand + walk) % n


def _host_layers(torch, fm, wl, weights):
    """Layer descriptors of `weights` with the canonical expert blobs in page-locked host memory."""
    hosts, descs = [], []
    for l, dl in enumerate(weights.layers):
        blobs = synth.expert_blobs(wl, l, 0, wl.n_experts + 1)
        h = torch.from_numpy(blobs.reshape(-1)).pin_memory()
        hosts.append(h)
        d = dl.desc()
        d["experts_dev"] = h.data_ptr()
        descs.append(fm.LayerDesc(**d))
    return hosts, descs


def _tokens(wl, n, start=0):
    from synth.gpu import tokens
    idx = list(range(start, start + n))
    return tokens(wl, idx, tie_free_subseeds(wl, 0, idx))


@pytest.mark.parametrize("wl", [TINY, RAGGED, TINY2, ZIPF], ids=lambda w: w.name)
@pytest.mark.parametrize("slots", ["2K", "E/2", "E"])
def test_cached_layer_is_bit_identical_and_counts_match_clock(torch, wl, slots):
    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights
    K, E = wl.top_k, wl.n_experts
    n_slots = {"2K": 2 * K, "E/2": max(2 * K, E // 2), "E": E}[slots]
    N = 48
    x = _tokens(wl, N)
    stream = torch.cuda.current_stream().cuda_stream
    def call(c, t, T, out, idx, w):
        # index / weight outputs of a call: their own [T][K] buffers (16-byte aligned)
        ic = torch.empty((T, K), dtype=torch.int32, device="cuda")
        wc = torch.empty((T, K), dtype=torch.float32, device="cuda")
        fm.fmoe_layer_forward(c, 0, x[t].data_ptr(), T, out[t].data_ptr(), ic.data_ptr(), wc.data_ptr(), stream)
        idx[t:t + T] = ic
        w[t:t + T] = wc

    with Model(wl) as m:
        want = torch.empty_like(x)
        widx = torch.empty((N, K), dtype=torch.int32, device="cuda")
        ww = torch.empty((N, K), dtype=torch.float32, device="cuda")
        for t in range(N):  # one token per call, the cached context's launch order
            call(m.ctx, t, 1, want, widx, ww)
        torch.cuda.synchronize()
    weights = DeviceWeights(wl)
    hosts, descs = _host_layers(torch, fm, wl, weights)
    _, ctx = fm.fmoe_create_cached(config_for(wl, 1, max_tokens=4), descs, n_slots, stream)
    try:
        for rnd in range(2):  # a second pass over the same tokens: warm cache
            got = torch.empty_like(x)
            gidx = torch.empty((N, K), dtype=torch.int32, device="cuda")
            gw = torch.empty((N, K), dtype=torch.float32, device="cuda")
            t = 0
            while t < N:  # calls of 1 and 3 tokens
                T = 1 if (t // 4) % 2 == 0 else min(3, N - t)
                call(ctx, t, T, got, gidx, gw)
                t += T
            st, word = fm.fmoe_poll_status(ctx, stream)
            assert st == 0 and word == 0
            assert np.array_equal(bf16_tensor_bits(got), bf16_tensor_bits(want)), rnd
            assert torch.equal(gidx, widx) and torch.equal(gw, ww), rnd
        hits, misses = fm.fmoe_cache_stats(ctx, stream)
    finally:
        fm.fmoe_destroy(ctx)
    model = ClockModel(n_slots)
    picks = widx.cpu().numpy()
    for _ in range(2):
        for t in range(N):
            model.step(0, [int(e) for e in picks[t]])
    assert hits + misses == 2 * N * K
    assert (hits, misses) == (model.hits, model.misses)
    if n_slots == E:  # everything fits: the second pass only hits
        assert misses == len({int(e) for e in picks.ravel()})


def test_cached_stack_is_bit_identical(torch):
    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights
    wl = STACK5
    K, L, T = wl.top_k, wl.n_layers, 3
    x = _tokens(wl, T, start=10)
    stream = torch.cuda.current_stream().cuda_stream
    with Model(wl) as m:
        want = torch.empty_like(x)
        m.fm.fmoe_stack_forward(m.ctx, 0, L, x.data_ptr(), T, want.data_ptr(), m.stream)
        torch.cuda.synchronize()
    weights = DeviceWeights(wl)
    hosts, descs = _host_layers(torch, fm, wl, weights)
    _, ctx = fm.fmoe_create_cached(config_for(wl, L, max_tokens=T), descs, 3 * K, stream)
    try:
        for rnd in range(3):
            got = torch.empty_like(x)
            fm.fmoe_stack_forward(ctx, 0, L, x.data_ptr(), T, got.data_ptr(), stream)
            st, word = fm.fmoe_poll_status(ctx, stream)
            assert st == 0 and word == 0
            assert np.array_equal(bf16_tensor_bits(got), bf16_tensor_bits(want)), rnd
        hits, misses = fm.fmoe_cache_stats(ctx, stream)
        assert hits + misses == 3 * L * T * K
        # unpacking reads the host copy (routed) or the HBM copy (shared)
        blob = fm.fmoe_expert_bytes(wl.hidden, wl.inter, wl.bits)
        dst = torch.empty(blob, dtype=torch.uint8, device="cuda")
        for e in (0, wl.n_experts - 1, -1):
            fm.fmoe_unpack_expert(ctx, 2, e, dst.data_ptr(), stream)
            torch.cuda.synchronize()
            ee = wl.n_experts if e < 0 else e
            assert np.array_equal(dst.cpu().numpy(), synth.expert_blob(wl, 2, ee)), e
    finally:
        fm.fmoe_destroy(ctx)


def test_cached_context_rejects_bad_use(torch):
    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights
    wl = TINY
    stream = torch.cuda.current_stream().cuda_stream
    weights = DeviceWeights(wl)
    cfg = config_for(wl, 1, max_tokens=4)
    device_descs = [fm.LayerDesc(**d) for d in weights.descs()]
    st, ctx = fm.fmoe_create_cached(cfg, device_descs, 8, stream, check=False)  # experts in device memory
    assert st == fm.FMOE_ERR_INVALID_ARG and ctx is None
    assert "page-locked" in fm.fmoe_last_error(None)
    hosts, descs = _host_layers(torch, fm, wl, weights)
    st, ctx = fm.fmoe_create_cached(cfg, descs, 2 * wl.top_k - 1, stream, check=False)
    assert st == fm.FMOE_ERR_INVALID_ARG and ctx is None
    _, ctx = fm.fmoe_create_cached(cfg, descs, 2 * wl.top_k, stream)
    try:
        x = _tokens(wl, 1)
        y = torch.empty((1, wl.hidden), dtype=torch.float32, device="cuda")
        st = fm.fmoe_expert_forward(ctx, 0, 1, x.data_ptr(), 1, y.data_ptr(), stream, check=False)
        assert st == fm.FMOE_ERR_UNSUPPORTED
    finally:
        fm.fmoe_destroy(ctx)
    with Model(wl) as m:
        with pytest.raises(fm.FmoeError):
            fm.fmoe_cache_stats(m.ctx, m.stream)
