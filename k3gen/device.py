"""Upload a workload's synthetic inputs to the GPU (plumbing only: generation
happens in k3gen, nothing here computes any part of the layer).

bf16 tensors are stored as int16 tensors holding the bf16 bit patterns.
"""
from __future__ import annotations

import numpy as np
import torch

import k3gen

_WEIGHTS = {}


class DeviceWeights:
    """Router, all E expert blobs (one slab) and the shared expert."""

    def __init__(self, cfg: k3gen.Config, seed: int = 0, device="cuda", batch: int = 32):
        self.cfg = cfg
        self.seed = seed
        self.w_router_host = k3gen.router(cfg, seed)
        self.w_router = torch.from_numpy(self.w_router_host).to(device)
        nb = cfg.blob_bytes
        self.blobs = torch.empty((cfg.E, nb), dtype=torch.uint8, device=device)
        pinned = torch.empty((min(batch, cfg.E), nb), dtype=torch.uint8).pin_memory()
        pn = pinned.numpy()
        for e0 in range(0, cfg.E, batch):
            n = min(batch, cfg.E - e0)
            for i in range(n):
                k3gen.expert_blob(cfg, e0 + i, seed, out=pn[i])
            self.blobs[e0:e0 + n].copy_(pinned[:n], non_blocking=False)
        self.blob_ptrs = torch.tensor([self.blobs[e].data_ptr() for e in range(cfg.E)],
                                      dtype=torch.int64, device=device)
        if cfg.ff_shared:
            wg, wu, wd = k3gen.shared(cfg, seed)
            self.shared_host = (wg, wu, wd)
            self.shared = tuple(torch.from_numpy(a.view(np.int16)).to(device) for a in (wg, wu, wd))
        else:
            self.shared_host = None
            self.shared = (None, None, None)

    def blob_host(self, e: int) -> np.ndarray:
        """Expert e's blob regenerated on the host (same bytes as on the device)."""
        return k3gen.expert_blob(self.cfg, e, self.seed)


def weights(cfg: k3gen.Config, seed: int = 0, device="cuda") -> DeviceWeights:
    """Device weights shared by every workload with the same layer shape."""
    key = (cfg.d, cfg.ff, cfg.E, cfg.ff_shared, cfg.scale_lo, cfg.scale_count, seed, str(device))
    w = _WEIGHTS.get(key)
    if w is None:
        w = DeviceWeights(cfg, seed, device)
        _WEIGHTS[key] = w
    return w


def release_all():
    _WEIGHTS.clear()
    torch.cuda.empty_cache()


class DeviceInputs:
    """Per-workload activations: x [T, d] (bf16 bits) and the router bias."""

    def __init__(self, cfg: k3gen.Config, seed: int = 0, device="cuda", T: int | None = None):
        self.cfg = cfg
        self.x_host = k3gen.hidden(cfg, seed, T)
        self.T = self.x_host.shape[0]
        self.x = torch.from_numpy(self.x_host.view(np.int16)).to(device)
        self.bias_host = k3gen.bias(cfg, seed)
        self.bias = None if self.bias_host is None else torch.from_numpy(self.bias_host).to(device)
