"""Seeded synthetic inputs shaped like the Flash-MoE model (test/bench infrastructure).

The Flash-MoE pages run a trained Qwen3.5-397B-A17B checkpoint; no weights or
datasets exist here, so every tensor is drawn from a counter-based generator
(SplitMix64, see ``synth_core.h``) with the distributions of the workloads
below.  The host library (``libsynth.so``, gcc) and the device generator
(``libsynth_cuda.so``, nvcc) produce identical bytes, so any expert of a
multi-GB weight set can be regenerated on the host for the oracle while the
GPU copy is generated in place.

This module holds no mixture-of-experts arithmetic: it draws numbers, rounds
them to bf16 and lays integer codes out in the canonical expert-blob format.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(HERE, "libsynth.so")
CUDA_LIB = os.path.join(HERE, "libsynth_cuda.so")
_lock = threading.Lock()
_host = None
_cuda = None

T_CODES, T_SCALE, T_BIAS, T_ROUTER, T_NORM, T_TOKEN = 1, 4, 7, 10, 11, 12


class ExpertParams(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint64), ("layer", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("bits", ctypes.c_int32), ("scale_lo", ctypes.c_double),
                ("scale_hi", ctypes.c_double), ("bias_lo", ctypes.c_double), ("bias_hi", ctypes.c_double)]


def _stale(out, srcs):
    return not os.path.exists(out) or os.path.getmtime(out) < max(os.path.getmtime(s) for s in srcs)


def build_host(force=False):
    srcs = [os.path.join(HERE, "synth.c"), os.path.join(HERE, "synth_core.h")]
    if force or _stale(HOST_LIB, srcs):
        tmp = HOST_LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c11",
                        "-o", tmp, srcs[0]], check=True)
        os.replace(tmp, HOST_LIB)
    return HOST_LIB


def build_cuda(force=False):
    srcs = [os.path.join(HERE, "synth_cuda.cu"), os.path.join(HERE, "synth_core.h")]
    if force or _stale(CUDA_LIB, srcs):
        tmp = CUDA_LIB + f".tmp{os.getpid()}"
        subprocess.run(["nvcc", "-O3", "-shared", "-Xcompiler", "-fPIC", "-fmad=false",
                        "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp, srcs[0]], check=True)
        os.replace(tmp, CUDA_LIB)
    return CUDA_LIB


def build(force=False):
    build_host(force)
    build_cuda(force)


def host():
    global _host
    with _lock:
        if _host is None:
            build_host()
            L = ctypes.CDLL(HOST_LIB)
            P, u64, u32, i64, dbl = (ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64,
                                     ctypes.c_double)
            L.synth_key_c.argtypes = [u64, u32, u32, u32]
            L.synth_key_c.restype = u64
            L.synth_draw_c.argtypes = [u64, u64]
            L.synth_draw_c.restype = u64
            L.synth_double_to_bf16_c.argtypes = [dbl]
            L.synth_double_to_bf16_c.restype = ctypes.c_uint16
            L.synth_blob_bytes_c.argtypes = [ctypes.POINTER(ExpertParams)]
            L.synth_blob_bytes_c.restype = i64
            L.synth_gen_experts.argtypes = [ctypes.POINTER(ExpertParams), ctypes.c_int, ctypes.c_int, P]
            L.synth_gen_normal_bf16.argtypes = [u64, u32, u32, u32, i64, dbl, dbl, P]
            L.synth_gen_uniform_bf16.argtypes = [u64, u32, u32, u32, i64, dbl, dbl, P]
            L.synth_gen_raw.argtypes = [u64, u32, u32, u32, i64, P]
            _host = L
    return _host


def cuda():
    global _cuda
    with _lock:
        if _cuda is None:
            build_cuda()
            L = ctypes.CDLL(CUDA_LIB)
            P = ctypes.c_void_p
            L.synth_cuda_gen_experts.argtypes = [ctypes.POINTER(ExpertParams), ctypes.c_int, ctypes.c_int, P, P]
            L.synth_cuda_gen_experts.restype = ctypes.c_int
            L.synth_cuda_gen_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                                     ctypes.c_uint32, ctypes.c_int64, ctypes.c_double,
                                                     ctypes.c_double, P, P]
            L.synth_cuda_gen_normal_bf16.restype = ctypes.c_int
            L.synth_cuda_gen_normal_rows_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                                          ctypes.c_uint32, ctypes.c_int, ctypes.c_int64,
                                                          ctypes.c_double, ctypes.c_double, P, P]
            L.synth_cuda_gen_normal_rows_bf16.restype = ctypes.c_int
            _cuda = L
    return _cuda


# --------------------------------------------------------------------------- workloads


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes and input distributions of one synthetic workload."""
    name: str
    hidden: int
    n_experts: int
    top_k: int
    inter: int
    bits: int
    n_layers: int
    tokens: int          # tokens per run (decode) or tokens per step (batched)
    steps: int           # batched steps (1 for batch-1 decode)
    norm: bool           # RMSNorm ahead of every layer
    zipf: float          # router-logit Zipf skew exponent (0 = none)
    seed: int
    scale_lo: float = 0.005
    scale_hi: float = 0.02
    bias_lo: float = -0.1
    bias_hi: float = 0.1
    router_std: float = 0.02
    x_std: float = 1.0
    norm_mean: float = 1.0
    norm_std: float = 0.02
    rms_eps: float = 1e-6

    @property
    def blob_bytes(self) -> int:
        return blob_bytes(self.hidden, self.inter, self.bits)

    def params(self, layer: int) -> ExpertParams:
        return ExpertParams(self.seed, layer, self.hidden, self.inter, self.bits, self.scale_lo,
                            self.scale_hi, self.bias_lo, self.bias_hi)


WORKLOADS = {
    # tiny single layer: H 256, 16 experts, top-2 + shared, I 128, 4-bit, seed 0
    "tiny": Workload("tiny", 256, 16, 2, 128, 4, 1, 1, 1, False, 0.0, 0),
    # one full-shape layer, batch-1 decode, 1000 seeded tokens
    "layer": Workload("layer", 4096, 512, 4, 1024, 4, 1, 1000, 1, False, 0.0, 1),
    # 24-layer 4-bit stack with RMSNorm + residual, 256 sequential tokens
    "stack4": Workload("stack4", 4096, 512, 4, 1024, 4, 24, 256, 1, True, 0.0, 2),
    # 60-layer 2-bit stack with RMSNorm + residual, 256 sequential tokens
    "stack2": Workload("stack2", 4096, 512, 4, 1024, 2, 60, 256, 1, True, 0.0, 3),
    # batched decode: 256 tokens per step, Zipf(1.1) router skew, 100 steps
    "batched": Workload("batched", 4096, 512, 4, 1024, 4, 1, 256, 100, False, 1.1, 4),
}


def blob_bytes(hidden, inter, bits) -> int:
    p = ExpertParams(0, 0, hidden, inter, bits, 0, 0, 0, 0)
    return int(host().synth_blob_bytes_c(ctypes.byref(p)))


def expert_blobs(wl: Workload, layer: int, first: int, count: int) -> np.ndarray:
    """Canonical blobs of experts first..first+count-1 of a layer (expert index
    n_experts is the shared expert), as a uint8 array [count, blob_bytes]."""
    out = np.empty((count, wl.blob_bytes), dtype=np.uint8)
    p = wl.params(layer)
    host().synth_gen_experts(ctypes.byref(p), first, count, out.ctypes.data_as(ctypes.c_void_p))
    return out


def expert_blob(wl: Workload, layer: int, expert: int) -> np.ndarray:
    return expert_blobs(wl, layer, expert, 1)[0]


def _normal(seed, layer, tensor, item, n, mean, std) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    host().synth_gen_normal_bf16(seed, layer, tensor, item, n, mean, std, out.ctypes.data_as(ctypes.c_void_p))
    return out


def router_weight(wl: Workload, layer: int) -> np.ndarray:
    """bf16 bits [E][H], N(0, router_std)."""
    return _normal(wl.seed, layer, T_ROUTER, 0, wl.n_experts * wl.hidden, 0.0, wl.router_std).reshape(
        wl.n_experts, wl.hidden)


def norm_weight(wl: Workload, layer: int) -> np.ndarray:
    """bf16 bits [H], N(norm_mean, norm_std)."""
    return _normal(wl.seed, layer, T_NORM, 0, wl.hidden, wl.norm_mean, wl.norm_std)


def token(wl: Workload, index: int, subseed: int = 0) -> np.ndarray:
    """bf16 bits [H] of token `index`, N(0, x_std); `subseed` selects a redraw."""
    return _normal(wl.seed, subseed, T_TOKEN, index, wl.hidden, 0.0, wl.x_std)


def raw(seed, layer, tensor, item, n) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    host().synth_gen_raw(seed, layer, tensor, item, n, out.ctypes.data_as(ctypes.c_void_p))
    return out


def zipf_bias(wl: Workload, layer: int) -> np.ndarray | None:
    """Per-expert router-logit bias -s*ln(rank) with ranks 1..E assigned by a
    seeded Fisher-Yates permutation (fp32 [E]); None when the workload has none."""
    if not wl.zipf:
        return None
    E = wl.n_experts
    r = raw(wl.seed, layer, T_ROUTER, 1, E)
    rank = np.arange(1, E + 1)
    for i in range(E - 1, 0, -1):
        j = int(r[i] % np.uint64(i + 1))
        rank[i], rank[j] = rank[j], rank[i]
    return np.array([-wl.zipf * math.log(float(k)) for k in rank], dtype=np.float32)


def double_to_bf16(v: float) -> int:
    return int(host().synth_double_to_bf16_c(float(v)))


# --------------------------------------------------------------------------- device side


def device_expert_blobs(wl: Workload, layer: int, first: int, count: int, dst_ptr: int, stream_ptr: int = 0):
    """Writes the same blobs as expert_blobs() into device memory at dst_ptr."""
    p = wl.params(layer)
    rc = cuda().synth_cuda_gen_experts(ctypes.byref(p), first, count, ctypes.c_void_p(dst_ptr),
                                       ctypes.c_void_p(stream_ptr))
    if rc != 0:
        raise RuntimeError(f"synth_cuda_gen_experts failed: cudaError {rc}")


def device_normal(seed, layer, tensor, item, n, mean, std, dst_ptr: int, stream_ptr: int = 0):
    rc = cuda().synth_cuda_gen_normal_bf16(seed, layer, tensor, item, n, mean, std, ctypes.c_void_p(dst_ptr),
                                           ctypes.c_void_p(stream_ptr))
    if rc != 0:
        raise RuntimeError(f"synth_cuda_gen_normal_bf16 failed: cudaError {rc}")


def device_router_weight(wl: Workload, layer: int, dst_ptr: int, stream_ptr: int = 0):
    device_normal(wl.seed, layer, T_ROUTER, 0, wl.n_experts * wl.hidden, 0.0, wl.router_std, dst_ptr, stream_ptr)


def device_norm_weight(wl: Workload, layer: int, dst_ptr: int, stream_ptr: int = 0):
    device_normal(wl.seed, layer, T_NORM, 0, wl.hidden, wl.norm_mean, wl.norm_std, dst_ptr, stream_ptr)


def device_token(wl: Workload, index: int, subseed: int, dst_ptr: int, stream_ptr: int = 0):
    device_normal(wl.seed, subseed, T_TOKEN, index, wl.hidden, 0.0, wl.x_std, dst_ptr, stream_ptr)


def device_token_range(wl: Workload, first: int, count: int, subseed: int, dst_ptr: int, stream_ptr: int = 0):
    """Tokens first..first+count-1 (bf16 rows of H) in one launch; same bytes as device_token."""
    rc = cuda().synth_cuda_gen_normal_rows_bf16(ctypes.c_uint64(wl.seed), ctypes.c_uint32(subseed),
                                                ctypes.c_uint32(T_TOKEN), ctypes.c_uint32(first), count,
                                                ctypes.c_int64(wl.hidden), ctypes.c_double(0.0),
                                                ctypes.c_double(wl.x_std), ctypes.c_void_p(dst_ptr),
                                                ctypes.c_void_p(stream_ptr))
    if rc != 0:
        raise RuntimeError(f"synth_cuda_gen_normal_rows_bf16 failed: cudaError {rc}")
