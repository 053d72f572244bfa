"""Helpers of the GPU parity tests: one layer call through the C ABI, and the
oracle's output for the same tokens (routed with the GPU's selection where
the oracle agrees that it is a valid top-k).  Comparison rules: parity.py."""
from __future__ import annotations

import numpy as np
import torch

from parity import check_topk_row


def lib():
    import mxfp4_routed_expert_softmax_b200 as m
    return m


def dims_of(cfg, flags=0):
    return lib().make_dims(cfg.d, cfg.ff, cfg.E, cfg.k, cfg.ff_shared, flags)


def run_layer(cfg, W, x, bias, T, flags=0, ptrs=None, ws_tokens=None):
    """y, idx, w of one k3moe_layer call (workspace sized for ws_tokens, by
    default T: the grouped path when T > 8)."""
    m = lib()
    dims = dims_of(cfg, flags)
    ws = m.new_workspace(dims, T if ws_tokens is None else ws_tokens)
    out32 = bool(flags & m.K3MOE_OUT_FP32)
    y = torch.empty((T, cfg.d), dtype=torch.float32 if out32 else torch.int16, device="cuda")
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    sg, su, sd = W.shared if not (flags & m.K3MOE_NO_SHARED) else (None, None, None)
    st = m.k3moe_layer(x, T, W.w_router, bias, W.blob_ptrs if ptrs is None else ptrs, sg, su, sd,
                       dims, y, idx, w, ws)
    m.check(st, "k3moe_layer")
    torch.cuda.synchronize()
    m.check(m.k3moe_device_status(ws), "device status")
    return y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def oracle_reference(orc, cfg, W, x_host, bias_host, gpu_idx, tokens, shared=True, renorm=False,
                     bias_select_only=False):
    """Oracle y for the given tokens, routed with the GPU's selection when the
    oracle agrees it is a valid top-k (else a problem is reported).  The
    routing variants: weights renormalised over the picks, the bias moving
    only the selection.  -> (y, problems, decisive count, probs, idx used,
    oracle weights at the GPU's picks)"""
    xs = x_host[tokens]
    logits, probs, idx_o, w_o = orc.route_variant(xs, W.w_router_host, bias_host, cfg.k, renorm=renorm,
                                                  bias_select_only=bias_select_only)
    scores = logits + bias_host.astype(np.float64) if (bias_select_only and bias_host is not None) else logits
    problems = []
    idx_use = np.empty_like(idx_o)
    n_decisive = 0
    for i, t in enumerate(tokens):
        decisive, pr = check_topk_row(scores[i], gpu_idx[t], cfg.k)
        n_decisive += decisive
        problems += [f"token {t}: {p}" for p in pr]
        idx_use[i] = gpu_idx[t]
    weight = np.take_along_axis(probs, idx_use.astype(np.int64), axis=1)
    if renorm:
        weight = weight / weight.sum(axis=1, keepdims=True)
    cache = {}
    slot_blobs = []
    for i in range(len(tokens)):
        for j in range(cfg.k):
            e = int(idx_use[i, j])
            if e not in cache:
                cache[e] = W.blob_host(e)
            slot_blobs.append(cache[e])
    sh = W.shared_host if shared else None
    y = orc.combine(xs, weight, slot_blobs, sh, cfg.d, cfg.ff)
    return y, problems, n_decisive, probs, idx_use, weight


def sample_tokens(T, n, seed=None):
    """n tokens of T (all when T <= n): the first, the last and a seeded draw."""
    if T <= n:
        return list(range(T))
    rng = np.random.default_rng(T if seed is None else seed)
    s = set(rng.choice(T, n - 2, replace=False).tolist()) | {0, T - 1}
    return sorted(s)


def last_group_of_busiest_expert(idx, group=32):
    """Tokens of the last group (of `group` tokens, in token order) of the
    expert that the most tokens selected: the grouped path's ragged tail
    where the most groups precede it."""
    e_all = idx.reshape(-1)
    counts = np.bincount(e_all)
    e = int(counts.argmax())
    toks = np.nonzero((idx == e).any(axis=1))[0]
    n = toks.size
    return toks[(n - 1) // group * group:].tolist(), e, n


def bf16_scale(x_bits, s, mask=None):
    """bf16 bits times 2^s (exact for results in bf16's normal range); only
    where mask is set when a mask is given."""
    f = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64) * (2.0 ** s)
    out = (f.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    if mask is None:
        return out
    return np.where(mask, out, x_bits).astype(np.uint16)
