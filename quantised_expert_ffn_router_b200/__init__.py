"""Python binding of libfmoe.so, the C-ABI mixture-of-experts decode library.

Argument marshalling only: every function forwards to the C entry point of
the same name in ``include/fmoe.h`` (device pointers and a CUDA stream handle
as plain integers).  All computation runs in the library's CUDA kernels; there
is no Python or CPU fallback, and importing this package fails loudly when the
library cannot be built or loaded.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

__all__ = [
    "FMOE_OK", "FMOE_ERR_INVALID_ARG", "FMOE_ERR_UNSUPPORTED", "FMOE_ERR_ALIGNMENT", "FMOE_ERR_CUDA",
    "FMOE_ERR_OOM", "FMOE_ERR_TIMEOUT", "FMOE_FLAG_FORCE_PER_TOKEN", "FMOE_FLAG_FORCE_GROUPED", "FMOE_FLAG_STACK_PER_LAYER",
    "FMOE_FLAG_DEBUG_SKIP_ROUTER_RELEASE", "Config", "LayerDesc", "FmoeError", "lib", "fmoe_expert_bytes",
    "fmoe_create", "fmoe_route", "fmoe_route_static", "fmoe_expert_forward", "fmoe_layer_forward", "fmoe_stack_forward",
    "fmoe_layer_forward_host", "fmoe_stack_forward_host", "fmoe_unpack_expert", "fmoe_poll_status", "fmoe_destroy", "fmoe_last_error", "EXPORTED_SYMBOLS",
    "fmoe_set_trace", "fmoe_trace_points", "fmoe_trace_layers", "fmoe_debug_set_epoch", "use_trace_build",
    "fmoe_create_cached", "fmoe_cache_stats",
]

FMOE_OK, FMOE_ERR_INVALID_ARG, FMOE_ERR_UNSUPPORTED, FMOE_ERR_ALIGNMENT = 0, 1, 2, 3
FMOE_ERR_CUDA, FMOE_ERR_OOM, FMOE_ERR_TIMEOUT = 4, 5, 6
FMOE_FLAG_FORCE_PER_TOKEN = 0x1
FMOE_FLAG_FORCE_GROUPED = 0x2
FMOE_FLAG_STACK_PER_LAYER = 0x4
FMOE_FLAG_DEBUG_SKIP_ROUTER_RELEASE = 0x100

EXPORTED_SYMBOLS = ["fmoe_expert_bytes", "fmoe_create", "fmoe_create_cached", "fmoe_cache_stats", "fmoe_route", "fmoe_route_static", "fmoe_expert_forward",
                    "fmoe_layer_forward", "fmoe_stack_forward", "fmoe_layer_forward_host", "fmoe_stack_forward_host",
                    "fmoe_unpack_expert", "fmoe_requant_4to2", "fmoe_set_gemm_events", "fmoe_set_trace",
                    "fmoe_trace_points", "fmoe_trace_layers", "fmoe_debug_set_epoch",
                    "fmoe_poll_status", "fmoe_destroy", "fmoe_last_error"]


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("bits", ctypes.c_int32), ("group", ctypes.c_int32),
                ("n_layers", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("rms_eps", ctypes.c_float),
                ("flags", ctypes.c_uint32), ("wait_timeout_us", ctypes.c_uint32)]


class LayerDesc(ctypes.Structure):
    _fields_ = [("router_w_dev", ctypes.c_void_p), ("router_bias_dev", ctypes.c_void_p),
                ("experts_dev", ctypes.c_void_p), ("norm_w_dev", ctypes.c_void_p)]


class FmoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"fmoe status {status}: {message}")
        self.status = status


_lock = threading.Lock()
_lib = None
_trace = False


def use_trace_build() -> None:
    """Loads libfmoe_trace.so (the same sources built with FMOE_TRACE, which
    records phase timestamps through fmoe_set_trace) instead of libfmoe.so.
    Must be called before the first library call of the process."""
    global _trace
    with _lock:
        if _lib is not None and not _trace:
            raise RuntimeError("the product library is already loaded")
        _trace = True


def lib():
    """The loaded libfmoe.so (built in-tree with nvcc when missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.LIB_TRACE if _trace else _build.LIB
            if _build.stale(trace=_trace):
                path = _build.build(trace=_trace)
            if not os.path.exists(path):
                raise ImportError(f"libfmoe.so not found at {path}")
            L = ctypes.CDLL(path)
            P, i32, u32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32
            L.fmoe_expert_bytes.argtypes = [i32, i32, i32]
            L.fmoe_expert_bytes.restype = ctypes.c_size_t
            L.fmoe_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(LayerDesc), P, ctypes.POINTER(P)]
            L.fmoe_create_cached.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(LayerDesc), ctypes.c_int64, P,
                                             ctypes.POINTER(P)]
            L.fmoe_cache_stats.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64)]
            L.fmoe_route.argtypes = [P, i32, P, i32, P, P, P]
            L.fmoe_route_static.argtypes = [P, i32, P, i32, P, P, P]
            L.fmoe_expert_forward.argtypes = [P, i32, i32, P, i32, P, P]
            L.fmoe_layer_forward.argtypes = [P, i32, P, i32, P, P, P, P]
            L.fmoe_stack_forward.argtypes = [P, i32, i32, P, i32, P, P]
            L.fmoe_layer_forward_host.argtypes = [P, i32, P, i32, P, P, P, P]
            L.fmoe_stack_forward_host.argtypes = [P, i32, i32, P, i32, P, P]
            L.fmoe_unpack_expert.argtypes = [P, i32, i32, P, P]
            L.fmoe_poll_status.argtypes = [P, P, ctypes.POINTER(u32)]
            L.fmoe_set_gemm_events.argtypes = [P, P]
            L.fmoe_requant_4to2.argtypes = [P, i32, i32, i32, P, P]
            L.fmoe_set_trace.argtypes = [P, P]
            L.fmoe_trace_points.argtypes = []
            L.fmoe_trace_layers.argtypes = []
            L.fmoe_debug_set_epoch.argtypes = [P, u32, P]
            L.fmoe_destroy.argtypes = [P]
            L.fmoe_last_error.argtypes = [P]
            L.fmoe_last_error.restype = ctypes.c_char_p
            for name in ("fmoe_create", "fmoe_create_cached", "fmoe_cache_stats", "fmoe_route", "fmoe_expert_forward", "fmoe_layer_forward",
                         "fmoe_stack_forward", "fmoe_layer_forward_host", "fmoe_stack_forward_host",
                         "fmoe_unpack_expert", "fmoe_poll_status", "fmoe_destroy", "fmoe_set_trace",
                         "fmoe_trace_points", "fmoe_trace_layers", "fmoe_debug_set_epoch"):
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def _check(ctx, status: int) -> int:
    if status != FMOE_OK:
        raise FmoeError(status, fmoe_last_error(ctx))
    return status


def _vp(x):
    return None if x is None or x == 0 else ctypes.c_void_p(int(x))


def fmoe_last_error(ctx=None) -> str:
    msg = lib().fmoe_last_error(_vp(ctx))
    return msg.decode() if msg else ""


def fmoe_expert_bytes(hidden: int, inter: int, bits: int) -> int:
    return int(lib().fmoe_expert_bytes(hidden, inter, bits))


def fmoe_create(cfg: Config, layers, stream: int = 0, *, check: bool = True):
    """Returns (status, ctx handle as int or None)."""
    arr = (LayerDesc * len(layers))(*layers)
    out = ctypes.c_void_p()
    st = lib().fmoe_create(ctypes.byref(cfg), arr, _vp(stream), ctypes.byref(out))
    if check:
        _check(None, st)
    return st, out.value


def fmoe_create_cached(cfg: Config, layers, cache_slots: int, stream: int = 0, *, check: bool = True):
    """Context whose routed experts stay in page-locked host memory (each
    layer's experts_dev a host pointer) behind an HBM cache of `cache_slots`
    expert slots.  Returns (status, ctx handle as int or None)."""
    arr = (LayerDesc * len(layers))(*layers)
    out = ctypes.c_void_p()
    st = lib().fmoe_create_cached(ctypes.byref(cfg), arr, ctypes.c_int64(cache_slots), _vp(stream), ctypes.byref(out))
    if check:
        _check(None, st)
    return st, out.value


def fmoe_cache_stats(ctx, stream=0):
    """(hits, misses) of a cached context's expert cache (synchronises `stream`)."""
    h, m = ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check(ctx, lib().fmoe_cache_stats(_vp(ctx), _vp(stream), ctypes.byref(h), ctypes.byref(m)))
    return int(h.value), int(m.value)


def fmoe_route(ctx, layer, x_dev, T, idx_dev, w_dev, stream=0, *, check=True) -> int:
    st = lib().fmoe_route(_vp(ctx), layer, _vp(x_dev), T, _vp(idx_dev), _vp(w_dev), _vp(stream))
    return _check(ctx, st) if check else st


def fmoe_route_static(ctx, layer, x_dev, T, idx_dev, w_dev, stream=0, *, check=True) -> int:
    st = lib().fmoe_route_static(_vp(ctx), layer, _vp(x_dev), T, _vp(idx_dev), _vp(w_dev), _vp(stream))
    return _check(ctx, st) if check else st


def fmoe_expert_forward(ctx, layer, expert, x_dev, T, y_dev, stream=0, *, check=True) -> int:
    st = lib().fmoe_expert_forward(_vp(ctx), layer, expert, _vp(x_dev), T, _vp(y_dev), _vp(stream))
    return _check(ctx, st) if check else st


def fmoe_layer_forward(ctx, layer, h_in_dev, T, h_out_dev, idx_out_dev=None, w_out_dev=None, stream=0, *,
                       check=True) -> int:
    st = lib().fmoe_layer_forward(_vp(ctx), layer, _vp(h_in_dev), T, _vp(h_out_dev), _vp(idx_out_dev),
                                  _vp(w_out_dev), _vp(stream))
    return _check(ctx, st) if check else st


def fmoe_stack_forward(ctx, layer_begin, layer_end, h_in_dev, T, h_out_dev, stream=0, *, check=True) -> int:
    st = lib().fmoe_stack_forward(_vp(ctx), layer_begin, layer_end, _vp(h_in_dev), T, _vp(h_out_dev), _vp(stream))
    return _check(ctx, st) if check else st


def fmoe_layer_forward_host(ctx, layer, h_in_host, T, h_out_host, idx_out_host=None, w_out_host=None, stream=0, *,
                            check=True) -> int:
    """fmoe_layer_forward on host buffers (addresses of page-locked memory)."""
    st = lib().fmoe_layer_forward_host(_vp(ctx), layer, _vp(h_in_host), T, _vp(h_out_host), _vp(idx_out_host),
                                       _vp(w_out_host), _vp(stream))
    return _check(ctx, st) if check else st


def fmoe_stack_forward_host(ctx, layer_begin, layer_end, h_in_host, T, h_out_host, stream=0, *, check=True) -> int:
    """fmoe_stack_forward on host buffers (addresses of page-locked memory)."""
    st = lib().fmoe_stack_forward_host(_vp(ctx), layer_begin, layer_end, _vp(h_in_host), T, _vp(h_out_host),
                                       _vp(stream))
    return _check(ctx, st) if check else st


def fmoe_unpack_expert(ctx, layer, expert, dst_dev, stream=0, *, check=True) -> int:
    st = lib().fmoe_unpack_expert(_vp(ctx), layer, expert, _vp(dst_dev), _vp(stream))
    return _check(ctx, st) if check else st


def fmoe_requant_4to2(src_ptr, n_blobs: int, hidden: int, inter: int, dst_ptr, stream=0) -> int:
    """Canonical 4-bit blobs at src_ptr -> canonical 2-bit blobs at dst_ptr."""
    return _check(None, lib().fmoe_requant_4to2(_vp(src_ptr), n_blobs, hidden, inter, _vp(dst_ptr), _vp(stream)))


def fmoe_set_gemm_events(ctx, handles=None) -> int:
    """Records the grouped GEMMs of later batched calls between 4 caller-owned
    cudaEvent_t handles (ints); None clears the hook."""
    if handles is None:
        return lib().fmoe_set_gemm_events(_vp(ctx), None)
    arr = (ctypes.c_void_p * 4)(*[int(h) for h in handles])
    return lib().fmoe_set_gemm_events(_vp(ctx), arr)


def fmoe_set_trace(ctx, trace_dev=None) -> int:
    """Phase timestamps of later fused-kernel launches into a uint64 device
    buffer [n_sm][fmoe_trace_layers()][fmoe_trace_points()] (trace build only);
    None clears the hook."""
    return _check(ctx, lib().fmoe_set_trace(_vp(ctx), _vp(trace_dev)))


def fmoe_trace_points() -> int:
    return lib().fmoe_trace_points()


def fmoe_trace_layers() -> int:
    return lib().fmoe_trace_layers()


def fmoe_debug_set_epoch(ctx, epoch: int, stream=0) -> int:
    """Test hook: sets the context's tag epoch (synchronises `stream`)."""
    return _check(ctx, lib().fmoe_debug_set_epoch(_vp(ctx), ctypes.c_uint32(epoch), _vp(stream)))


def fmoe_poll_status(ctx, stream=0):
    """Returns (status, raw device status word)."""
    word = ctypes.c_uint32(0)
    st = lib().fmoe_poll_status(_vp(ctx), _vp(stream), ctypes.byref(word))
    return st, word.value


def fmoe_destroy(ctx) -> int:
    return lib().fmoe_destroy(_vp(ctx))
