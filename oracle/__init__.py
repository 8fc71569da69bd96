"""Plain double-precision CPU oracle of the Flash-MoE mixture-of-experts decode step.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg (and its ``--impl reference`` arm) are the only
callers.  The product library never imports this package and shares no code
with it.

The arithmetic lives in ``oracle.c`` (built into ``liboracle.so`` with gcc);
this module marshals numpy arrays and composes the steps of one layer in the
order the Flash-MoE pages give them (the Hysen Labs page "Flash-MoE: Running a
397B Parameter Model on a Laptop", section "How the SSD expert streaming
pipeline works": normalisation and routing in the second command buffer,
softmax and top-K on the host, then the third command buffer runs the experts
and combines their outputs).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")
_SOURCES = [os.path.join(HERE, "oracle.c"), os.path.join(HERE, "oracle.h")]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (double precision, no FP contraction)."""
    newest = max(os.path.getmtime(s) for s in _SOURCES)
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= newest:
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11",
           "-o", tmp, os.path.join(HERE, "oracle.c"), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(LIB_PATH)
            P = ctypes.c_void_p
            i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            L.orc_bf16_value.argtypes = [ctypes.c_uint16]
            L.orc_bf16_value.restype = dbl
            L.orc_round_bf16.argtypes = [dbl]
            L.orc_round_bf16.restype = ctypes.c_uint16
            L.orc_blob_bytes.argtypes = [i32, i32, i32]
            L.orc_blob_bytes.restype = i64
            L.orc_weight.argtypes = [P, i32, i32, i32, i32, i32, i32]
            L.orc_weight.restype = dbl
            L.orc_rmsnorm.argtypes = [P, P, i32, dbl, P]
            L.orc_router_logits.argtypes = [P, P, P, i32, i32, P]
            L.orc_topk.argtypes = [P, i32, i32, P, P, P]
            L.orc_expert.argtypes = [P, i32, i32, i32, P, P, P, P, P]
            L.orc_combine.argtypes = [P, P, P, P, i32, i32, P, P]
            L.orc_requant_4to2.argtypes = [P, i32, i32, P]
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def bf16_value(bits: int) -> float:
    return lib().orc_bf16_value(int(bits) & 0xFFFF)


def round_bf16(v: float) -> int:
    return int(lib().orc_round_bf16(float(v)))


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact values of a uint16 array of bf16 bit patterns (vectorised widening)."""
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def blob_bytes(hidden: int, inter: int, bits: int) -> int:
    return int(lib().orc_blob_bytes(hidden, inter, bits))


def weight(blob: np.ndarray, hidden: int, inter: int, bits: int, m: int, r: int, c: int) -> float:
    blob = _c(blob, np.uint8)
    return lib().orc_weight(_ptr(blob), hidden, inter, bits, m, r, c)


def rmsnorm(h: np.ndarray, w: np.ndarray | None, eps: float) -> np.ndarray:
    h = _c(h, np.uint16)
    w = _c(w, np.uint16)
    z = np.empty_like(h)
    lib().orc_rmsnorm(_ptr(h), _ptr(w), h.size, float(eps), _ptr(z))
    return z


def router_logits(wr: np.ndarray, bias: np.ndarray | None, z: np.ndarray) -> np.ndarray:
    wr = _c(wr, np.uint16)
    z = _c(z, np.uint16)
    bias = _c(bias, np.float32)
    E, H = wr.shape
    out = np.empty(E, dtype=np.float32)
    lib().orc_router_logits(_ptr(wr), _ptr(bias), _ptr(z), H, E, _ptr(out))
    return out


def topk(logits: np.ndarray, k: int):
    """Returns (idx int32 [k], w float64 [k], p float64 [E])."""
    logits = _c(logits, np.float32)
    E = logits.size
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    p = np.empty(E, dtype=np.float64)
    lib().orc_topk(_ptr(logits), E, k, _ptr(idx), _ptr(w), _ptr(p))
    return idx, w, p


def expert(blob: np.ndarray, hidden: int, inter: int, bits: int, z: np.ndarray):
    """Returns (y [hidden], g [inter], u [inter], a [inter]) as float64."""
    blob = _c(blob, np.uint8)
    z = _c(z, np.uint16)
    g = np.empty(inter)
    u = np.empty(inter)
    a = np.empty(inter)
    y = np.empty(hidden)
    lib().orc_expert(_ptr(blob), hidden, inter, bits, _ptr(z), _ptr(g), _ptr(u), _ptr(a), _ptr(y))
    return y, g, u, a


def combine(h: np.ndarray, w: np.ndarray, y_routed: np.ndarray, y_shared: np.ndarray):
    """Returns (out_f64 [H], out_bf16 uint16 [H])."""
    h = _c(h, np.uint16)
    w = _c(w, np.float64)
    y_routed = _c(y_routed, np.float64)
    y_shared = _c(y_shared, np.float64)
    H = h.size
    k = w.size
    out64 = np.empty(H)
    out = np.empty(H, dtype=np.uint16)
    lib().orc_combine(_ptr(h), _ptr(w), _ptr(y_routed), _ptr(y_shared), H, k, _ptr(out64), _ptr(out))
    return out64, out


def layer_forward(h, *, router_w, router_bias, norm_w, eps, top_k, hidden, inter, bits, blob_of):
    """One mixture-of-experts layer for one token.

    ``blob_of(e)`` returns the canonical blob of expert e (0..E-1 routed, E the
    shared expert); it is only asked for the K selected experts and the shared
    one.  Steps, in the order of that page's pipeline: norm -> router -> softmax
    and top-K -> expert forward (K routed + shared) -> combine into the residual.
    Returns a dict with z, logits, idx, w, y (routed, [K][H]), y_shared, out_f64
    and out (bf16 bits).
    """
    h = _c(h, np.uint16)
    z = rmsnorm(h, norm_w, eps) if norm_w is not None else h.copy()
    logits = router_logits(router_w, router_bias, z)
    idx, w, _ = topk(logits, top_k)
    E = router_w.shape[0]
    ys = np.stack([expert(blob_of(int(e)), hidden, inter, bits, z)[0] for e in idx])
    y_sh = expert(blob_of(E), hidden, inter, bits, z)[0]
    out64, out = combine(h, w, ys, y_sh)
    return dict(z=z, logits=logits, idx=idx, w=w, y=ys, y_shared=y_sh, out_f64=out64, out=out)


def requant_4to2(blob: np.ndarray, hidden: int, inter: int) -> np.ndarray:
    """Canonical 2-bit blob refitted from a canonical 4-bit blob (orc_requant_4to2)."""
    blob = _c(blob, np.uint8)
    out = np.zeros(blob_bytes(hidden, inter, 2), dtype=np.uint8)
    lib().orc_requant_4to2(_ptr(blob), hidden, inter, _ptr(out))
    return out


def topk_gaps(logits: np.ndarray, k: int) -> float:
    """Smallest gap between adjacent logits among the k+1 largest (tie margin)."""
    s = np.sort(np.asarray(logits, dtype=np.float64))[::-1][: k + 1]
    return float(np.min(s[:-1] - s[1:]))
