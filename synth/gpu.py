"""Device-resident synthetic weights and tokens (test/bench infrastructure).

Allocates torch CUDA tensors and fills them with the seeded generator's bytes
(the same bytes the host generator gives the oracle).  Holds no
mixture-of-experts arithmetic and does not call the product library.
"""
from __future__ import annotations

import torch

from . import (Workload, device_expert_blobs, device_norm_weight, device_router_weight, device_token,
               device_token_range, zipf_bias)


class DeviceLayer:
    def __init__(self, wl: Workload, layer: int, stream: int):
        E, H = wl.n_experts, wl.hidden
        self.router = torch.empty((E, H), dtype=torch.bfloat16, device="cuda")
        device_router_weight(wl, layer, self.router.data_ptr(), stream)
        self.experts = torch.empty(((E + 1) * wl.blob_bytes,), dtype=torch.uint8, device="cuda")
        device_expert_blobs(wl, layer, 0, E + 1, self.experts.data_ptr(), stream)
        self.norm = None
        if wl.norm:
            self.norm = torch.empty((H,), dtype=torch.bfloat16, device="cuda")
            device_norm_weight(wl, layer, self.norm.data_ptr(), stream)
        b = zipf_bias(wl, layer)
        self.bias = None if b is None else torch.from_numpy(b).to("cuda")

    def desc(self) -> dict:
        return dict(router_w_dev=self.router.data_ptr(),
                    router_bias_dev=0 if self.bias is None else self.bias.data_ptr(),
                    experts_dev=self.experts.data_ptr(),
                    norm_w_dev=0 if self.norm is None else self.norm.data_ptr())


class DeviceWeights:
    """All layers of a workload on the current CUDA device."""

    def __init__(self, wl: Workload, n_layers: int | None = None):
        self.wl = wl
        stream = torch.cuda.current_stream().cuda_stream
        n = wl.n_layers if n_layers is None else n_layers
        self.layers = [DeviceLayer(wl, l, stream) for l in range(n)]
        torch.cuda.current_stream().synchronize()

    def descs(self) -> list[dict]:
        return [l.desc() for l in self.layers]


def tokens(wl: Workload, indices, subseeds=None) -> torch.Tensor:
    """bf16 [len(indices)][H] device tensor of tokens `indices` (redraw `subseeds`)."""
    stream = torch.cuda.current_stream().cuda_stream
    out = torch.empty((len(indices), wl.hidden), dtype=torch.bfloat16, device="cuda")
    idx = [int(t) for t in indices]
    if subseeds is None and len(idx) > 1 and idx == list(range(idx[0], idx[0] + len(idx))):
        device_token_range(wl, idx[0], len(idx), 0, out.data_ptr(), stream)
        return out
    for r, t in enumerate(indices):
        s = 0 if subseeds is None else int(subseeds[r])
        device_token(wl, int(t), s, out[r].data_ptr(), stream)
    return out
