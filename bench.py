#!/usr/bin/env python
"""Benchmark of the batch-1 mixture-of-experts decode step on B200.

Default workload ("layer"): one full-shape layer -- hidden 4096, 512 experts,
top-4 renormalised + 1 shared expert, SwiGLU intermediate 1024, 4-bit group-64
affine codes with bf16 scale/bias, bf16 router N(0, 0.02) -- decoding 1000
seeded tokens x ~ N(0, 1) one at a time.  One step = one token through the
whole hot path (router GEMV, softmax, top-K, K+1 dequantising SwiGLU experts,
combine) = one fused kernel launch.  The weights stay resident in HBM; L2 is
flushed (a 256 MB write, then a 256 MB read) before every timed step, so the router and shared
expert are read from HBM as they would be inside a multi-layer model; each
step is timed with CUDA events on the launching stream and the flush is not.

Other workloads: "stack4" (24 layers, 4-bit, RMSNorm + residual, 256 tokens)
and "stack2" (60 layers, 2-bit), one step = one token through every layer
(per-step weight traffic ~1 GB, far above L2, so no flush).

``--impl reference`` times the plain double-precision CPU oracle on the same
workload, metric and unit (the pages' own engine runs only on Apple Metal).

Multi-GPU (torchrun): replicas only -- every rank decodes its own copy of the
workload with no collective on the data path; ranks meet at a barrier and
the step time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "kernel_traffic.json")
CSRC = os.path.join(ROOT, "quantised_expert_ffn_router_b200", "csrc")
FALLBACK_HBM_GBS = 6650.0


# kernels one batched layer step launches: norm, router, logit sum, top-K,
# permute, input prep, GEMV fragments, gate/up GEMM (tcgen05), gate/up GEMV,
# activation prep, GEMV fragments, down GEMM (tcgen05), down GEMV, combine
BATCHED_LAUNCHES = 14


# the sources each timed kernel is compiled from: a DRAM capture stays valid
# (roofline.traffic) until one of them changes
KERNEL_SOURCES = {"layer": ["fmoe_decode.cu", "fmoe_internal.h"],
                  "batched": ["fmoe_grouped_tc.cu", "fmoe_batched.cu", "fmoe_internal.h"]}


def kernel_source_sha(key: str) -> str:
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[key]):
        h.update(name.encode())
        h.update(open(os.path.join(CSRC, name), "rb").read())
    return h.hexdigest()[:16]


def hbm_peak():
    try:
        p = json.load(open(PEAKS_PATH))
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def layer_bytes(wl: synth.Workload) -> int:
    """Algorithmic bytes of one token through one layer: router weights, K routed
    + 1 shared expert blobs, norm weight, token in and out (bf16)."""
    b = wl.n_experts * wl.hidden * 2 + (wl.top_k + 1) * wl.blob_bytes + 2 * wl.hidden * 2
    if wl.norm:
        b += wl.hidden * 2
    return b


# ----------------------------------------------------------------------------- clocks


class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML every few ms."""

    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sync_boost", 0x40: "sw_thermal_slowdown",
             0x80: "hw_thermal_slowdown", 0x100: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int):
        super().__init__(daemon=True)
        self.samples = []
        self.stop_flag = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def run(self):
        if not self.ok:
            return
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM), int(get_reasons(self.h))))
            except Exception:
                pass
            time.sleep(0.005)

    def summary(self):
        self.stop_flag.set()
        self.join(timeout=1)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.NAMES.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


class Flush:
    """Evicts L2 (126 MB on B200) between timed steps: a 256 MB write, then a
    256 MB read of another buffer, so the timed kernel finds neither its own
    weights in L2 nor the write's dirty lines (which a real decode step, whose
    neighbours mostly read weights, would not leave behind either)."""

    def __init__(self, torch):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(64 << 20, dtype=torch.int32, device="cuda")

    def __call__(self, i):
        self.w.fill_(i & 0xFF)
        self.r.max()


# ----------------------------------------------------------------------------- oracle (CPU)


def oracle_tokens_per_s(wl: synth.Workload, n_tokens_max: int, budget_s: float):
    """Times the CPU oracle on up to n_tokens_max tokens of the workload (first
    layer for the single-layer workload, every layer for stacks), stopping after
    budget_s seconds.  Returns (tokens/s, tokens done, threads, seconds)."""
    import oracle
    layers = wl.n_layers
    cache = {}

    def host_layer(l):
        if l not in cache:
            cache[l] = dict(router=synth.router_weight(wl, l), bias=synth.zipf_bias(wl, l),
                            norm=synth.norm_weight(wl, l) if wl.norm else None, blobs={})
        return cache[l]

    def blob_of(l):
        d = host_layer(l)

        def get(e):
            if e not in d["blobs"]:
                d["blobs"][e] = synth.expert_blob(wl, l, e)
            return d["blobs"][e]
        return get

    # routing pass (not timed) to pre-generate the experts the sample touches
    n_tokens_max = max(1, n_tokens_max)
    xs = [synth.token(wl, t) for t in range(n_tokens_max)]
    if layers == 1:
        d = host_layer(0)
        for x in xs:
            z = oracle.rmsnorm(x, d["norm"], wl.rms_eps) if d["norm"] is not None else x
            idx, _, _ = oracle.topk(oracle.router_logits(d["router"], d["bias"], z), wl.top_k)
            for e in list(idx) + [wl.n_experts]:
                blob_of(0)(int(e))
    threads = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    done = 0
    for x in xs:
        h = x
        for l in range(layers):
            d = host_layer(l)
            r = oracle.layer_forward(h, router_w=d["router"], router_bias=d["bias"], norm_w=d["norm"],
                                     eps=wl.rms_eps, top_k=wl.top_k, hidden=wl.hidden, inter=wl.inter, bits=wl.bits,
                                     blob_of=blob_of(l))
            h = r["out"]
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, threads, dt


def run_reference(args, wl, rank):
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    n = warmup + steps
    tps_w, _, _, _ = oracle_tokens_per_s(wl, max(1, warmup), 1e9) if warmup else (0, 0, 0, 0)
    tps, done, threads, dt = oracle_tokens_per_s(wl, steps, args.cpu_seconds * 4)
    line = {
        "impl": "reference",
        "metric": metric_name(wl), "value": tps, "unit": "tokens/s", "n_gpus": args.gpus, "steps": done,
        "warmup": warmup, "ms_per_step": 1e3 * dt / max(done, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, shaped like the pages' model)",
        "config": config_dict(wl, flushed=False, cpu=True),
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{done} tokens of workload '{wl.name}' ({wl.n_layers} layer(s) each)"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm


def metric_name(wl):
    return "MoE decode tokens/s and us/layer; expert+router HBM GB/s as fraction of peak"


def config_dict(wl, flushed, cpu=False):
    batched = wl.name == "batched"
    return {"workload": wl.name,
            "shape": f"H{wl.hidden} E{wl.n_experts} top{wl.top_k}+1shared I{wl.inter} {wl.bits}-bit g64",
            "layers": wl.n_layers, "tokens": wl.tokens * (wl.steps if batched else 1),
            "batch": wl.tokens if batched else 1, "norm": wl.norm,
            **({"router_bias": f"Zipf(s={wl.zipf}) over a seeded expert ranking"} if wl.zipf else {}),
            "l2": "n/a (CPU oracle)" if cpu else ("flushed (256 MB write + 256 MB read) before every timed step" if flushed else
                                                  "per-step weight traffic far above L2 (no flush)"),
            "parallelism": "replicas"}


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(ws, value: float, device: str = "cuda") -> float:
    """The largest of every rank's value (timings are taken as the slowest rank)."""
    if ws == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ws: int, units_per_rank: int, max_ms: float) -> float:
    """Whole-job units/s: every rank's units over the slowest rank's time."""
    return ws * units_per_rank / (max_ms / 1e3)


def run_gpu(args, wl, ws, rank, local):
    line = measure_gpu(args, wl, ws, rank, local, args.steps, args.warmup, args.e2e_steps,
                       cpu_baseline=ws == 1 and not args.no_cpu_baseline)
    if line is None:
        return 0
    if wl.name == "layer" and ws == 1 and not args.no_workloads:
        # the other full-size workloads, each on its own weights (freed before the next)
        line["workloads"] = {}
        for name, steps in (("stack4", 64), ("stack2", 32), ("batched", 30)):
            import torch
            torch.cuda.empty_cache()
            w = measure_gpu(args, synth.WORKLOADS[name], ws, rank, local, steps, 3, min(steps, 16), cpu_baseline=False)
            line["workloads"][name] = workload_summary(w)
        import torch
        torch.cuda.empty_cache()
        line["workloads"]["cached"] = measure_cached()
    print(json.dumps(line), flush=True)
    return 0


def measure_cached(steps: int = 200) -> dict:
    """Host-resident experts behind the HBM expert cache (fmoe_create_cached),
    on the single-layer shape: us/layer and hit rate with a cold cache (2K
    slots, uniform routing), with a Zipf(1.1)-skewed router and 64 slots, and
    with every expert cached; the host->HBM rate the misses stream at, next to
    a plain pinned host->device copy of the same link."""
    import ctypes
    import dataclasses

    import torch

    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceLayer, tokens

    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    out = {}
    # the link: one pinned 256 MB host->device copy, timed on the stream
    hb = torch.empty(256 << 20, dtype=torch.uint8, pin_memory=True)
    db = torch.empty_like(hb, device="cuda")
    for _ in range(3):
        db.copy_(hb, non_blocking=True)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(5):
        db.copy_(hb, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize()
    out["link_h2d_gbs"] = 5 * hb.numel() / (a.elapsed_time(b) * 1e-3) / 1e9
    del hb, db
    base = synth.WORKLOADS["layer"]
    cases = (("cold", base, 2 * base.top_k), ("zipf", dataclasses.replace(base, name="layer_zipf", zipf=1.1), 64),
             ("warm", base, base.n_experts))
    for name, wl, n_slots in cases:
        E, K = wl.n_experts, wl.top_k
        blob = wl.blob_bytes
        host = torch.empty((E + 1) * blob, dtype=torch.uint8, pin_memory=True)
        p = wl.params(0)
        synth.host().synth_gen_experts(ctypes.byref(p), 0, E + 1, ctypes.c_void_p(host.data_ptr()))
        dl = DeviceLayer(wl, 0, sp)
        d = dl.desc()
        d["experts_dev"] = host.data_ptr()
        del dl.experts  # routed experts are read from host memory only
        cfg = fm.Config(wl.hidden, E, K, wl.inter, wl.bits, 64, 1, 1, wl.rms_eps, 0, 0)
        _, ctx = fm.fmoe_create_cached(cfg, [fm.LayerDesc(**d)], n_slots, sp)
        X = tokens(wl, range(steps))
        Y = torch.empty_like(X)
        n_warm = steps if name == "warm" else 8  # warm: every token once, so every expert it picks is cached
        for i in range(n_warm):
            fm.fmoe_layer_forward(ctx, 0, X[i].data_ptr(), 1, Y[i].data_ptr(), None, None, sp)
        h0, m0 = fm.fmoe_cache_stats(ctx, sp)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(steps):
            fm.fmoe_layer_forward(ctx, 0, X[i].data_ptr(), 1, Y[i].data_ptr(), None, None, sp)
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        h1, m1 = fm.fmoe_cache_stats(ctx, sp)
        st, word = fm.fmoe_poll_status(ctx, sp)
        if st != 0:
            raise RuntimeError(f"device status 0x{word:x} (cached {name})")
        fm.fmoe_destroy(ctx)
        hits, misses = h1 - h0, m1 - m0
        out[name] = {"cache_slots": n_slots, "router": "Zipf(s=1.1)" if wl.zipf else "uniform",
                     "us_per_layer": 1e3 * ms / steps, "tokens_per_s": steps / (ms * 1e-3),
                     "hit_rate": hits / max(hits + misses, 1), "hits": hits, "misses": misses,
                     "host_gbs": misses * blob / (ms * 1e-3) / 1e9}
        del host, dl, X, Y
        torch.cuda.empty_cache()
    cold, warm = out["cold"], out["warm"]
    if cold["misses"] > 0:
        # what a missed expert adds to a layer, and the rate that implies
        per_miss_us = (cold["us_per_layer"] - warm["us_per_layer"]) / (cold["misses"] / steps)
        out["us_per_missed_expert"] = per_miss_us
        out["missed_expert_gbs"] = base.blob_bytes / (per_miss_us * 1e-6) / 1e9
    out["shape"] = "H4096 E512 top4+1shared I1024 4-bit g64, batch 1, one layer"
    out["steps"] = steps
    return out


def workload_summary(w: dict) -> dict:
    """The fields of a workload's bench line kept in the headline's `workloads` object."""
    keep = ("value", "unit", "steps", "warmup", "ms_per_step", "us_per_layer", "hbm_gbs", "hbm_frac", "roofline",
            "e2e", "gpu_launches", "clocks", "dtype", "config", "step_us_p10_p50_p90")
    out = {k: w[k] for k in keep if k in w}
    if "batched" in w:
        out["batched"] = w["batched"]
    return out


def measure_gpu(args, wl, ws, rank, local, steps, warmup, e2e_steps, cpu_baseline):
    """One workload's bench line (rank 0; None on other ranks)."""
    import torch

    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights, tokens

    torch.cuda.set_device(local)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    weights = DeviceWeights(wl)
    descs = [fm.LayerDesc(**d) for d in weights.descs()]
    batched = wl.name == "batched"
    B = wl.tokens if batched else 1          # tokens per step
    L = wl.n_layers
    stacked = L > 1
    # stacks: one launch per token through every layer, or (--stack-per-layer) one per layer
    per_layer = stacked and args.stack_per_layer
    flags = fm.FMOE_FLAG_STACK_PER_LAYER if per_layer else 0
    cfg = fm.Config(wl.hidden, wl.n_experts, wl.top_k, wl.inter, wl.bits, 64, wl.n_layers, B, wl.rms_eps, flags, 0)
    _, ctx = fm.fmoe_create(cfg, descs, sp)
    n_batches = wl.steps if batched else wl.tokens   # distinct inputs cycled through
    X = tokens(wl, range(n_batches * B)).view(n_batches, B, wl.hidden)
    OUT = torch.empty_like(X)
    IDX = torch.zeros((n_batches, B, wl.top_k), dtype=torch.int32, device="cuda")

    def step(i, x_ptr=None, out_ptr=None):
        x_ptr = X[i % n_batches].data_ptr() if x_ptr is None else x_ptr
        out_ptr = OUT[i % n_batches].data_ptr() if out_ptr is None else out_ptr
        if stacked:
            fm.fmoe_stack_forward(ctx, 0, L, x_ptr, B, out_ptr, sp)
        else:
            fm.fmoe_layer_forward(ctx, 0, x_ptr, B, out_ptr, IDX[i % n_batches].data_ptr() if batched else None,
                                  None, sp)

    # a batched step streams ~0.5 GB of expert weights, far above L2: no flush
    flush = Flush(torch) if not (stacked or batched) else None

    def maybe_flush(i):
        if flush is not None:
            flush(i)

    for i in range(warmup):
        maybe_flush(i)
        step(i)
    torch.cuda.synchronize()
    st, word = fm.fmoe_poll_status(ctx, sp)
    if st != 0:
        raise RuntimeError(f"device status 0x{word:x} after warm-up")

    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    # batched: the library records these around its two grouped GEMM launches
    # (recorded once here so that the handles exist)
    gemm_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)] if batched else None
    if batched:
        for evs in gemm_ev:
            for e in evs:
                e.record(stream)
        torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    barrier(ws)
    torch.cuda.synchronize()
    sampler.start()
    for i in range(steps):
        maybe_flush(i)
        if batched:
            fm.fmoe_set_gemm_events(ctx, [e.cuda_event for e in gemm_ev[i]])
        ev0[i].record(stream)
        step(i)
        ev1[i].record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    if batched:
        fm.fmoe_set_gemm_events(ctx, None)
        gemm_ms = [statistics.mean(e[2 * k].elapsed_time(e[2 * k + 1]) for e in gemm_ev) for k in range(2)]
    clocks = sampler.summary()
    step_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    total_ms = max_over_ranks(ws, sum(step_ms))
    st, word = fm.fmoe_poll_status(ctx, sp)
    if st != 0:
        raise RuntimeError(f"device status 0x{word:x} after timing")

    # warm (no flush) reference number for the single layer
    warm_us = None
    if not (stacked or batched):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(steps):
            step(i)
        b.record(stream)
        torch.cuda.synchronize()
        warm_us = 1e3 * a.elapsed_time(b) / steps

    # end to end through the public API with host buffers (pinned), copies timed
    e2e_steps = min(steps, e2e_steps)
    # one library call per step on page-locked host buffers: it enqueues the
    # input copy, the layer (or stack) and the output copy on the stream
    x_host = X[:min(n_batches, e2e_steps)].cpu().pin_memory()
    out_host = torch.empty_like(x_host).pin_memory()
    e2e_ms, call_us = [], []
    for i in range(e2e_steps):
        maybe_flush(i)
        j = i % len(x_host)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        c0 = time.perf_counter()
        if stacked:
            fm.fmoe_stack_forward_host(ctx, 0, L, x_host[j].data_ptr(), B, out_host[j].data_ptr(), sp)
        else:
            fm.fmoe_layer_forward_host(ctx, 0, x_host[j].data_ptr(), B, out_host[j].data_ptr(), None, None, sp)
        call_us.append(1e6 * (time.perf_counter() - c0))
        b.record(stream)
        stream.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_total = max_over_ranks(ws, sum(e2e_ms))
    # where the end-to-end time goes: the same step as three separately timed
    # parts (copy in, device call, copy out) with the stream's own copies
    parts = []
    xd, od = torch.empty_like(X[0]), torch.empty_like(OUT[0])
    for i in range(min(e2e_steps, 50)):
        maybe_flush(i)
        j = i % len(x_host)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        xd.copy_(x_host[j], non_blocking=True)
        ev[1].record(stream)
        step(i, xd.data_ptr(), od.data_ptr())
        ev[2].record(stream)
        out_host[j].copy_(od, non_blocking=True)
        ev[3].record(stream)
        stream.synchronize()
        parts.append([ev[k].elapsed_time(ev[k + 1]) for k in range(3)])
    e2e_parts_us = [1e3 * statistics.mean(p[k] for p in parts) for k in range(3)]
    del xd, od
    fm.fmoe_destroy(ctx)
    del weights, X, OUT, x_host, out_host

    if rank != 0:
        return None
    ms_per_step = total_ms / steps
    tps = job_throughput(ws, steps * B, total_ms)
    us_layer = 1e3 * ms_per_step / L
    bytes_launch = layer_bytes(wl)
    tensor = None
    if batched:
        # per step: router + every distinct selected expert + the shared one, tokens in and out
        idx_h = IDX.cpu().numpy()
        uniq = [len(set(idx_h[i % n_batches].ravel().tolist())) for i in range(steps)]
        del IDX
        bytes_launch = (wl.n_experts * wl.hidden * 2 + (statistics.mean(uniq) + 1) * wl.blob_bytes
                        + 2 * B * wl.hidden * 2)
        flops = 2 * B * (wl.top_k + 1) * 3 * wl.hidden * wl.inter + 2 * B * wl.hidden * wl.n_experts
        # the grouped GEMMs, timed on the launching stream: weights of every
        # selected expert once, inputs read and outputs written once
        P = B * (wl.top_k + 1)
        tb = 16 * 64 * wl.bits // 8 + 64
        gu_w = (wl.inter // 8) * (wl.hidden // 64) * tb
        dn_w = (wl.hidden // 16) * (wl.inter // 64) * tb
        ne = statistics.mean(uniq) + 1
        gu_bytes = ne * gu_w + P * wl.hidden * 2 + P * wl.inter * 4
        dn_bytes = ne * dn_w + P * wl.inter * 2 + P * wl.hidden * 4
        gu_flops = 2 * P * 2 * wl.inter * wl.hidden
        tensor = {"flops_per_step": flops, "achieved_tflops": flops / (ms_per_step * 1e-3) / 1e12,
                  "unique_experts_per_step": statistics.mean(uniq),
                  "gate_up_gemm": {"kernel": f"gate/up phase: bt_gv_frag_kernel, bt_tc_gemm_kernel<{wl.bits}, true>, "
                                             f"bt_gemv_kernel<{wl.bits}, true>", "us": 1e3 * gemm_ms[0],
                                   "algorithmic_bytes": gu_bytes, "gbs": gu_bytes / (gemm_ms[0] * 1e-3) / 1e9,
                                   "tflops": gu_flops / (gemm_ms[0] * 1e-3) / 1e12},
                  "down_gemm": {"kernel": f"down phase: bt_gv_frag_kernel, bt_tc_gemm_kernel<{wl.bits}, false>, "
                                          f"bt_gemv_kernel<{wl.bits}, false>", "us": 1e3 * gemm_ms[1],
                                "algorithmic_bytes": dn_bytes, "gbs": dn_bytes / (gemm_ms[1] * 1e-3) / 1e9,
                                "tflops": gu_flops / 2 / (gemm_ms[1] * 1e-3) / 1e12}}
    achieved = bytes_launch / (us_layer * 1e-6) / 1e9
    peak, peak_kind = hbm_peak()
    traffic = None
    try:
        tr = json.load(open(TRAFFIC_PATH))
        key = f"{wl.name}"
        if key in KERNEL_SOURCES and tr.get("source_sha", {}).get(key) == kernel_source_sha(key) \
                and key in tr.get("bytes_per_launch", {}):
            traffic = tr["bytes_per_launch"][key]
    except Exception:
        traffic = None
    line = {
        "metric": metric_name(wl), "value": tps, "unit": "tokens/s", "n_gpus": ws, "steps": steps,
        "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": ("exact integer codes x fp16 inputs on tcgen05, fp32 accumulate + fp32 scale/bias (bf16 I/O)"
                                       if batched else "fp16 tensor-core MAC of exact integer codes, fp32 accumulate (bf16 I/O)"),
        "data": "synthetic (seeded, shaped like the pages' model; random weights)",
        "config": {**config_dict(wl, flushed=not stacked),
                   **({"launch": "one per layer" if per_layer else "one per token through every layer"}
                      if stacked else {})},
        "us_per_layer": us_layer, "hbm_gbs": achieved, "hbm_frac": achieved / peak,
        "roofline": ({"bound": "hbm", "achieved": tensor["gate_up_gemm"]["gbs"], "peak": peak, "unit": "GB/s",
                      "frac": tensor["gate_up_gemm"]["gbs"] / peak, "traffic": traffic, "peak_source": peak_kind,
                      "kernel": tensor["gate_up_gemm"]["kernel"],
                      "algorithmic_bytes_per_launch": tensor["gate_up_gemm"]["algorithmic_bytes"]} if batched else
                     {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                      "traffic": traffic, "peak_source": peak_kind,
                      "kernel": f"decode_kernel<{wl.bits}, {'true' if stacked and not per_layer else 'false'}>",
                      "algorithmic_bytes_per_launch": bytes_launch}),
        "step_us_p10_p50_p90": [1e3 * q for q in statistics.quantiles(step_ms, n=10)[0::4]] if steps >= 10 else None,
        "warm_l2_us_per_layer": warm_us,
        "e2e": {"value": job_throughput(ws, e2e_steps * B, e2e_total), "unit": "tokens/s",
                "h2d_bytes_per_step": B * wl.hidden * 2, "d2h_bytes_per_step": B * wl.hidden * 2,
                "us_per_step": 1e3 * e2e_total / e2e_steps,
                "path": ("page-locked buffers: input read over the link by a stage-in kernel, output written "
                         "to host memory by the fused kernel" if not batched else
                         "one copy-engine transfer each way around the grouped path"),
                "host_call_us": statistics.median(call_us),
                "breakdown_copy_engine_us": {"h2d": e2e_parts_us[0], "device": e2e_parts_us[1],
                                             "d2h": e2e_parts_us[2]}},
        "gpu_launches": steps * (BATCHED_LAUNCHES if batched else (L if per_layer or not stacked else 1)),
        "clocks": clocks,
    }
    if tensor is not None:
        line["batched"] = tensor
    if cpu_baseline:
        tps_cpu, done, threads, dt = oracle_tokens_per_s(wl, 400, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tps_cpu, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"{done} tokens of workload '{wl.name}' ({L} layer(s) each), "
                                          f"{dt:.1f} s"}
    return line


# phase timestamps the trace build records per block and layer (fmoe_set_trace)
TRACE_POINTS = [(0, "start"), (1, "router copies issued"), (2, "input z ready"),
                (7, "block's router rows published"), (14, "block's shared units published"),
                (3, "every logit seen (producer)"), (4, "top-K done"), (5, "first routed copy issued"),
                (6, "every gate/up copy issued"), (8, "first routed gate/up chunk started"),
                (9, "block's last routed unit published"), (15, "first down job started"),
                (10, "first activations current"), (11, "last down job done"), (12, "combine done"),
                (13, "block exit")]


def run_trace(args, wl):
    """Per-phase timeline of the fused kernel from the trace build: for each
    recorded point, the median over steps of its median and latest time over
    blocks, in microseconds after the earliest block start of the launch."""
    import numpy as np
    import torch

    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceWeights, tokens
    fm.use_trace_build()
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    weights = DeviceWeights(wl)
    L = wl.n_layers
    cfg = fm.Config(wl.hidden, wl.n_experts, wl.top_k, wl.inter, wl.bits, 64, L, 1, wl.rms_eps, 0, 0)
    _, ctx = fm.fmoe_create(cfg, [fm.LayerDesc(**d) for d in weights.descs()], sp)
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    NP, NLt = fm.fmoe_trace_points(), fm.fmoe_trace_layers()
    buf = torch.zeros((n_sm, NLt, NP), dtype=torch.int64, device="cuda")
    fm.fmoe_set_trace(ctx, buf.data_ptr())
    n_tok = min(wl.tokens, 64)
    X = tokens(wl, range(n_tok))
    OUT = torch.empty_like(X)
    flush = Flush(torch) if L == 1 else None
    steps, warmup = args.steps, args.warmup
    recs = []
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    event_us = []
    for i in range(warmup + steps):
        if flush is not None:
            flush(i)
        buf.zero_()
        ev0.record(stream)
        if L > 1:
            fm.fmoe_stack_forward(ctx, 0, L, X[i % n_tok].data_ptr(), 1, OUT[i % n_tok].data_ptr(), sp)
        else:
            fm.fmoe_layer_forward(ctx, 0, X[i % n_tok].data_ptr(), 1, OUT[i % n_tok].data_ptr(), None, None, sp)
        ev1.record(stream)
        torch.cuda.synchronize()
        if i >= warmup:
            recs.append(buf.cpu().numpy().astype(np.float64))
            event_us.append(1e3 * ev0.elapsed_time(ev1))
    st, word = fm.fmoe_poll_status(ctx, sp)
    fm.fmoe_destroy(ctx)
    if st != 0:
        raise RuntimeError(f"device status 0x{word:x}")
    table = {}
    for layer in range(min(L, NLt)):
        rows = []
        for k, name in TRACE_POINTS:
            if k == 13 and layer > 0:
                continue
            med, late = [], []
            for r in recs:
                t0 = r[:, 0, 0][r[:, 0, 0] > 0].min()
                v = r[:, layer if k != 13 else 0, k]
                v = v[v > 0]
                if v.size:
                    med.append((np.median(v) - t0) / 1e3)
                    late.append((v.max() - t0) / 1e3)
            if med:
                rows.append({"point": name, "median_us": round(float(np.median(med)), 3),
                             "latest_us": round(float(np.median(late)), 3), "blocks": int(v.size)})
        table[f"layer{layer}"] = rows
    for layer, rows in table.items():
        print(f"# {wl.name} {layer}: median over {steps} launches (event time {statistics.median(event_us):.2f} us)")
        for r in rows:
            print(f"#   {r['point']:<48s} median block {r['median_us']:8.3f} us   latest block {r['latest_us']:8.3f} us")
    print(json.dumps({"trace": wl.name, "steps": steps, "event_us_median": statistics.median(event_us),
                      "phases": table}), flush=True)
    return 0


# fp32/integer operations per weight of the requantisation kernel: code
# extraction, int-to-float and fma in both passes, min/max, subtract, multiply,
# round, clamp and packing
REQUANT_OPS_PER_WEIGHT = 16


def run_requant(args):
    """4-bit -> 2-bit requantisation of one full layer's 513 expert blobs
    (H 4096, I 1024), timed with CUDA events; one GPU."""
    import torch

    import quantised_expert_ffn_router_b200 as fm
    from synth.gpu import DeviceLayer
    wl = synth.WORKLOADS["layer"]
    stream = torch.cuda.current_stream()
    layer = DeviceLayer(wl, 0, stream.cuda_stream)
    n = wl.n_experts + 1
    out = torch.empty(n * fm.fmoe_expert_bytes(wl.hidden, wl.inter, 2), dtype=torch.uint8, device="cuda")
    steps = args.steps or 20
    for _ in range(max(args.warmup, 3)):
        fm.fmoe_requant_4to2(layer.experts.data_ptr(), n, wl.hidden, wl.inter, out.data_ptr(), stream.cuda_stream)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    for a, b in evs:
        a.record(stream)
        fm.fmoe_requant_4to2(layer.experts.data_ptr(), n, wl.hidden, wl.inter, out.data_ptr(), stream.cuda_stream)
        b.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.summary()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    in_bytes = n * wl.blob_bytes
    out_bytes = out.numel()
    gbs = (in_bytes + out_bytes) / (ms * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()
    weights = n * 3 * wl.hidden * wl.inter
    # issue peak: 148 SMs x 128 lanes x the SM clock seen
    alu_peak = 148 * 128 * (clocks.get("sm_mhz") or 1965) * 1e6 / 1e12
    alu = weights * REQUANT_OPS_PER_WEIGHT / (ms * 1e-3) / 1e12
    line = {"metric": "4-bit -> 2-bit expert requantisation (one full layer, 513 blobs)", "value": gbs,
            "unit": "GB/s (bytes read + written)", "n_gpus": 1, "steps": steps, "warmup": max(args.warmup, 3),
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
            "data": "synthetic (seeded)", "config": {"workload": "requant", "shape": "H4096 I1024 513 blobs"},
            "roofline": {"bound": "alu", "achieved": alu, "peak": alu_peak, "unit": "T ops/s", "frac": alu / alu_peak,
                         "ops_per_weight": REQUANT_OPS_PER_WEIGHT, "hbm_gbs": gbs, "hbm_frac": gbs / peak,
                         "hbm_peak_source": peak_kind},
            "gpu_launches": steps, "clocks": clocks}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["layer", "stack4", "stack2", "tiny", "batched", "requant"], default="layer")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stack-per-layer", action="store_true",
                    help="stacks: one launch per layer instead of one per token (the multi-layer kernel)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="layer workload: skip the stack4 / stack2 / batched entries of the `workloads` object")
    ap.add_argument("--trace", action="store_true",
                    help="per-phase timeline of the fused kernel from the trace build (not a bench line)")
    args = ap.parse_args(argv)
    if args.workload == "requant":
        return run_requant(args)
    wl = synth.WORKLOADS[args.workload]
    if args.trace:
        args.steps = args.steps or 50
        return run_trace(args, wl)
    if args.steps is None:
        args.steps = {"layer": 3000, "stack4": 256, "stack2": 256, "tiny": 1000, "batched": 100}[args.workload]
    args.warmup = max(args.warmup, 3)
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, wl, rank)
    ws, rank, local = dist_setup(args)
    try:
        return run_gpu(args, wl, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
