"""The host-buffer entry points (fmoe_layer_forward_host,
fmoe_stack_forward_host) against the device-pointer calls: results must be
bit-identical, for one token, several tokens (token by token and on the
grouped path) and a multi-layer stack, with the expert indices and weights,
and with the input and output in one host buffer.  Page-locked buffers take
the path without copy-engine transfers (input read over the link by a
stage-in kernel, outputs written to host memory by the fused kernel);
pageable buffers take the copies."""
import dataclasses

import numpy as np
import pytest

import synth
from moe_cases import Model, tie_free_subseeds

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]
STACK5 = dataclasses.replace(TINY, name="hoststack5", n_layers=5, norm=True, seed=51)


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


def _pinned(torch, t):
    return torch.empty(t.shape, dtype=t.dtype, pin_memory=True)


@pytest.mark.parametrize("T", [1, 3, 8])
def test_layer_host_equals_device(torch, T):
    wl = TINY
    x = _x(wl, T, start=20)
    with Model(wl) as m:
        out = torch.empty_like(x)
        idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), w.data_ptr(), m.stream)
        xh = _pinned(torch, x)
        xh.copy_(x.cpu())
        oh, ih, wh = _pinned(torch, out), _pinned(torch, idx), _pinned(torch, w)
        m.fm.fmoe_layer_forward_host(m.ctx, 0, xh.data_ptr(), T, oh.data_ptr(), ih.data_ptr(), wh.data_ptr(),
                                     m.stream)
        torch.cuda.synchronize()
        st, word = m.fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == 0, hex(word)
        assert torch.equal(oh.view(torch.int16), out.cpu().view(torch.int16))
        assert torch.equal(ih, idx.cpu())
        assert torch.equal(wh, w.cpu())
        # buffers at an offset inside larger page-locked allocations
        big_in = torch.empty((2 * T, wl.hidden), dtype=x.dtype, pin_memory=True)
        big_out = torch.zeros((3 * T, wl.hidden), dtype=x.dtype, pin_memory=True)
        big_in[T:].copy_(x.cpu())
        m.fm.fmoe_layer_forward_host(m.ctx, 0, big_in[T:].data_ptr(), T, big_out[T:2 * T].data_ptr(), None, None,
                                     m.stream)
        torch.cuda.synchronize()
        assert torch.equal(big_out[T:2 * T].view(torch.int16), out.cpu().view(torch.int16))
        assert not big_out[:T].view(torch.int16).any() and not big_out[2 * T:].view(torch.int16).any()
        # input and output in one host buffer: the staging makes that safe
        m.fm.fmoe_layer_forward_host(m.ctx, 0, xh.data_ptr(), T, xh.data_ptr(), None, None, m.stream)
        torch.cuda.synchronize()
        assert torch.equal(xh.view(torch.int16), out.cpu().view(torch.int16))


@pytest.mark.parametrize("T", [1, 3])
def test_layer_host_pageable_equals_device(torch, T):
    wl = TINY
    x = _x(wl, T, start=60)
    with Model(wl) as m:
        out = torch.empty_like(x)
        idx = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, wl.top_k), dtype=torch.float32, device="cuda")
        m.fm.fmoe_layer_forward(m.ctx, 0, x.data_ptr(), T, out.data_ptr(), idx.data_ptr(), w.data_ptr(), m.stream)
        xh = x.cpu()  # pageable
        oh, ih, wh = torch.empty_like(xh), torch.empty_like(idx.cpu()), torch.empty_like(w.cpu())
        m.fm.fmoe_layer_forward_host(m.ctx, 0, xh.data_ptr(), T, oh.data_ptr(), ih.data_ptr(), wh.data_ptr(),
                                     m.stream)
        torch.cuda.synchronize()
        st, word = m.fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == 0, hex(word)
        assert torch.equal(oh.view(torch.int16), out.cpu().view(torch.int16))
        assert torch.equal(ih, idx.cpu()) and torch.equal(wh, w.cpu())


def test_stack_host_equals_device(torch):
    wl = STACK5
    x = _x(wl, 2, start=30)
    with Model(wl) as m:
        out = torch.empty_like(x)
        m.fm.fmoe_stack_forward(m.ctx, 0, wl.n_layers, x.data_ptr(), 2, out.data_ptr(), m.stream)
        xh, oh = _pinned(torch, x), _pinned(torch, x)
        xh.copy_(x.cpu())
        m.fm.fmoe_stack_forward_host(m.ctx, 0, wl.n_layers, xh.data_ptr(), 2, oh.data_ptr(), m.stream)
        m.fm.fmoe_stack_forward_host(m.ctx, 1, 4, xh.data_ptr(), 2, xh.data_ptr(), m.stream)
        part = torch.empty_like(x)
        m.fm.fmoe_stack_forward(m.ctx, 1, 4, x.data_ptr(), 2, part.data_ptr(), m.stream)
        torch.cuda.synchronize()
        st, word = m.fm.fmoe_poll_status(m.ctx, m.stream)
        assert st == 0, hex(word)
        assert torch.equal(oh.view(torch.int16), out.cpu().view(torch.int16))
        assert torch.equal(xh.view(torch.int16), part.cpu().view(torch.int16))


def test_host_calls_reject_bad_arguments(torch):
    import quantised_expert_ffn_router_b200 as fm
    wl = TINY
    with Model(wl) as m:
        h = _pinned(torch, torch.empty((2, wl.hidden), dtype=torch.bfloat16))
        assert fm.fmoe_layer_forward_host(m.ctx, 0, None, 1, h.data_ptr(), check=False) == fm.FMOE_ERR_INVALID_ARG
        assert fm.fmoe_layer_forward_host(m.ctx, 0, h.data_ptr(), 1, None, check=False) == fm.FMOE_ERR_INVALID_ARG
        assert fm.fmoe_layer_forward_host(m.ctx, 1, h.data_ptr(), 1, h.data_ptr(), check=False) == \
            fm.FMOE_ERR_INVALID_ARG
        assert fm.fmoe_layer_forward_host(m.ctx, 0, h.data_ptr(), 257, h.data_ptr(), check=False) == \
            fm.FMOE_ERR_INVALID_ARG
        assert fm.fmoe_stack_forward_host(m.ctx, 0, 2, h.data_ptr(), 1, h.data_ptr(), check=False) == \
            fm.FMOE_ERR_INVALID_ARG
        assert fm.fmoe_layer_forward_host(m.ctx, 0, None, 0, None, check=False) == fm.FMOE_OK
