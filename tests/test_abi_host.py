"""The C-ABI library on the host: it builds, loads, exports every entry point
include/fmoe.h declares, and rejects bad arguments with a status code before
any CUDA call (so these run without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

import oracle
import quantised_expert_ffn_router_b200 as fm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "fmoe.h")).read()
    return sorted(set(re.findall(r"FMOE_API\s+[\w\s\*]+?\b(fmoe_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(fm.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    L = fm.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", fm.lib()._name], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (fmoe_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_expert_bytes_matches_layout():
    assert fm.fmoe_expert_bytes(4096, 1024, 4) == 7077888
    assert fm.fmoe_expert_bytes(4096, 1024, 2) == 3932160
    for H, I, b in [(256, 128, 4), (320, 192, 2), (64, 64, 4)]:
        assert fm.fmoe_expert_bytes(H, I, b) == oracle.blob_bytes(H, I, b)
    assert fm.fmoe_expert_bytes(100, 64, 4) == 0
    assert fm.fmoe_expert_bytes(256, 128, 3) == 0


def _cfg(**kw):
    base = dict(hidden=256, n_experts=16, top_k=2, inter=128, bits=4, group=64, n_layers=1, max_tokens=8,
                rms_eps=1e-6, flags=0, wait_timeout_us=0)
    base.update(kw)
    return fm.Config(**base)


def _layer(router=0x1000, experts=0x2000, bias=0, norm=0):
    return fm.LayerDesc(router, bias, experts, norm)


@pytest.mark.parametrize("kw,status", [
    (dict(hidden=100), fm.FMOE_ERR_INVALID_ARG),
    (dict(hidden=0), fm.FMOE_ERR_INVALID_ARG),
    (dict(inter=96), fm.FMOE_ERR_INVALID_ARG),
    (dict(top_k=17), fm.FMOE_ERR_INVALID_ARG),
    (dict(top_k=0), fm.FMOE_ERR_INVALID_ARG),
    (dict(bits=3), fm.FMOE_ERR_INVALID_ARG),
    (dict(bits=8), fm.FMOE_ERR_INVALID_ARG),
    (dict(group=32), fm.FMOE_ERR_INVALID_ARG),
    (dict(n_experts=0), fm.FMOE_ERR_INVALID_ARG),
    (dict(n_layers=0), fm.FMOE_ERR_INVALID_ARG),
    (dict(max_tokens=-1), fm.FMOE_ERR_INVALID_ARG),
    (dict(rms_eps=float("nan")), fm.FMOE_ERR_INVALID_ARG),
    (dict(top_k=9, n_experts=32), fm.FMOE_ERR_UNSUPPORTED),
    (dict(hidden=8192), fm.FMOE_ERR_UNSUPPORTED),
    (dict(inter=8192), fm.FMOE_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_config(kw, status):
    st, ctx = fm.fmoe_create(_cfg(**kw), [_layer()], 0, check=False)
    assert st == status and ctx is None
    assert fm.fmoe_last_error(None)


def test_create_rejects_bad_layers():
    st, ctx = fm.fmoe_create(_cfg(), [_layer(router=0)], 0, check=False)
    assert st == fm.FMOE_ERR_INVALID_ARG and ctx is None
    st, ctx = fm.fmoe_create(_cfg(), [_layer(experts=0)], 0, check=False)
    assert st == fm.FMOE_ERR_INVALID_ARG
    for bad in (dict(router=0x1001), dict(experts=0x2008), dict(bias=0x3004), dict(norm=0x4002)):
        st, ctx = fm.fmoe_create(_cfg(), [_layer(**bad)], 0, check=False)
        assert st == fm.FMOE_ERR_ALIGNMENT, bad
    assert "aligned" in fm.fmoe_last_error(None)


def test_create_rejects_null_arguments():
    L = fm.lib()
    out = ctypes.c_void_p()
    assert L.fmoe_create(None, None, None, ctypes.byref(out)) == fm.FMOE_ERR_INVALID_ARG
    cfg = _cfg()
    assert L.fmoe_create(ctypes.byref(cfg), None, None, ctypes.byref(out)) == fm.FMOE_ERR_INVALID_ARG


def test_calls_on_invalid_context_fail_cleanly():
    bogus = 0xDEAD0
    assert fm.fmoe_layer_forward(bogus, 0, 0x1000, 1, 0x2000, check=False) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_route(bogus, 0, 0x1000, 1, 0x2000, 0x3000, check=False) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_expert_forward(bogus, 0, 0, 0x1000, 1, 0x2000, check=False) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_stack_forward(bogus, 0, 1, 0x1000, 1, 0x2000, check=False) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_layer_forward_host(bogus, 0, 0x1000, 1, 0x2000, check=False) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_stack_forward_host(bogus, 0, 1, 0x1000, 1, 0x2000, check=False) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_unpack_expert(bogus, 0, 0, 0x1000, check=False) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_poll_status(bogus)[0] == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_destroy(bogus) == fm.FMOE_ERR_INVALID_ARG
    assert fm.fmoe_destroy(None) == fm.FMOE_ERR_INVALID_ARG
    assert "destroyed" in fm.fmoe_last_error(bogus)
