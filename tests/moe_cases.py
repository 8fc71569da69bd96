"""Helpers shared by the GPU parity tests: contexts over synthetic workloads,
tie-free token selection (decided by the oracle on the host) and error metrics."""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle
import synth

TIE_GAP = 1e-3       # minimum gap between adjacent logits among the K+1 largest
REL_L2_TOL = 2e-3    # per-token relative L2 bound on outputs
W_TOL = 1e-5         # absolute bound on router weights


def config_for(wl: synth.Workload, n_layers: int, flags: int = 0, max_tokens: int = 256, timeout_us: int = 0):
    import quantised_expert_ffn_router_b200 as fm
    return fm.Config(wl.hidden, wl.n_experts, wl.top_k, wl.inter, wl.bits, 64, n_layers, max_tokens,
                     wl.rms_eps, flags, timeout_us)


class Model:
    """A context over a workload's device weights (layers 0..n_layers-1)."""

    def __init__(self, wl: synth.Workload, n_layers: int | None = None, flags: int = 0, timeout_us: int = 0):
        import torch

        import quantised_expert_ffn_router_b200 as fm
        from synth.gpu import DeviceWeights
        self.fm = fm
        self.wl = wl
        self.weights = DeviceWeights(wl, n_layers)
        n = len(self.weights.layers)
        descs = [fm.LayerDesc(**d) for d in self.weights.descs()]
        self.stream = torch.cuda.current_stream().cuda_stream
        _, self.ctx = fm.fmoe_create(config_for(wl, n, flags, timeout_us=timeout_us), descs, self.stream)

    def close(self):
        if self.ctx:
            self.fm.fmoe_destroy(self.ctx)
            self.ctx = None

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()


def tie_free_subseeds(wl: synth.Workload, layer: int, indices, gap: float = TIE_GAP, router_w=None):
    """For each token index, the first redraw whose oracle router logits have
    all gaps among the K+1 largest at least `gap` (layers without norm)."""
    wr = synth.router_weight(wl, layer) if router_w is None else router_w
    bias = synth.zipf_bias(wl, layer)
    norm = synth.norm_weight(wl, layer) if wl.norm else None
    out = []
    for t in indices:
        for s in range(64):
            x = synth.token(wl, int(t), s)
            z = oracle.rmsnorm(x, norm, wl.rms_eps) if norm is not None else x
            if oracle.topk_gaps(oracle.router_logits(wr, bias, z), wl.top_k) >= gap:
                out.append(s)
                break
        else:
            raise RuntimeError("no tie-free redraw found")
    return out


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def bf16_tensor_bits(t) -> np.ndarray:
    """uint16 numpy array of a bf16 torch tensor's bit patterns."""
    import torch
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


@dataclasses.dataclass
class OracleLayer:
    """Lazy per-layer host data for the oracle."""
    wl: synth.Workload
    layer: int

    def __post_init__(self):
        self.router = synth.router_weight(self.wl, self.layer)
        self.bias = synth.zipf_bias(self.wl, self.layer)
        self.norm = synth.norm_weight(self.wl, self.layer) if self.wl.norm else None
        self._blobs = {}

    def blob(self, e: int) -> np.ndarray:
        if e not in self._blobs:
            self._blobs[e] = synth.expert_blob(self.wl, self.layer, e)
        return self._blobs[e]

    def forward(self, h_bits: np.ndarray) -> dict:
        wl = self.wl
        return oracle.layer_forward(h_bits, router_w=self.router, router_bias=self.bias, norm_w=self.norm,
                                    eps=wl.rms_eps, top_k=wl.top_k, hidden=wl.hidden, inter=wl.inter, bits=wl.bits,
                                    blob_of=self.blob)
