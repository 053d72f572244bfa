"""k3moe_layer_residual: RMSNorm of the residual stream before the layer and
the residual add after it (a norm launch and the down pass's epilogue, or fused
into the one-launch kernel), against the oracle's
statement of the block: h_out = h + layer(RNE_bf16(RMSNorm(h))).  Tokens whose
top-k is a near tie under the oracle's logits (relative k / k+1 gap <= 1e-5)
are left out, since the kernel's fp32 normalisation may round an element of
x to the other bf16 neighbour and so pick the other expert."""
import numpy as np
import pytest
import torch

import k3gen
from gpu_helpers import dims_of, sample_tokens
from k3gen import device as kdev
from parity import G1_TOL, TOPK_REL_GAP, g1_error, rel_gap

pytestmark = pytest.mark.gpu

m = pytest.importorskip("mxfp4_routed_expert_softmax_b200") if torch.cuda.is_available() else None

SMALL = k3gen.Config("small", d=512, ff=256, E=64, k=8, ff_shared=192, T=0, bias="normal")
EPS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    kdev.release_all()


def oracle_block(orc, cfg, W, h, bias, g, tokens):
    """h + layer(RMSNorm(h)) for the given tokens, fp64, and which of them
    have a decisive top-k."""
    x = orc.rmsnorm(h[tokens], g, EPS)
    lg, probs, idx, wt = orc.route(x, W.w_router_host, bias, cfg.k)
    decisive = []
    for i in range(len(tokens)):
        srt = np.sort(lg[i])[::-1]
        decisive.append(cfg.k == cfg.E or rel_gap(srt[cfg.k - 1], srt[cfg.k]) > TOPK_REL_GAP)
    blobs = {}
    slot = []
    for i in range(len(tokens)):
        for j in range(cfg.k):
            e = int(idx[i, j])
            if e not in blobs:
                blobs[e] = W.blob_host(e)
            slot.append(blobs[e])
    y = orc.combine(x, wt, slot, W.shared_host, cfg.d, cfg.ff)
    return orc.residual_add(h[tokens], y), np.array(decisive)


# one_launch: the decode passes as one cooperative launch (K3MOE_ONE_LAUNCH)
# instead of the default norm + router + gate/up + down launches
@pytest.mark.parametrize("cfg,T,ws_tokens,one_launch", [
    (k3gen.CONFIGS["tiny"], 4, 4, False), (SMALL, 8, 8, False), (SMALL, 13, 8, False),
    (k3gen.CONFIGS["k3_decode"], 1, 1, False), (k3gen.CONFIGS["k3_decode_t8"], 8, 8, False),
    (k3gen.CONFIGS["tiny"], 64, 64, False), (SMALL, 40, 40, False),
    (SMALL, 13, 8, True), (k3gen.CONFIGS["k3_decode"], 1, 1, True), (k3gen.CONFIGS["k3_decode_t8"], 8, 8, True)])
def test_layer_residual_matches_oracle(orc, cfg, T, ws_tokens, one_launch):
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    g = k3gen.norm_weights(cfg)
    gd = torch.from_numpy(g.view(np.int16)).cuda()
    dims = dims_of(cfg, m.K3MOE_OUT_FP32 | (m.K3MOE_ONE_LAUNCH if one_launch else 0))
    ws = m.new_workspace(dims, ws_tokens)
    out = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
    m.check(m.k3moe_layer_residual(inp.x, T, gd, EPS, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims,
                                   out, ws), "k3moe_layer_residual")
    torch.cuda.synchronize()
    m.check(m.k3moe_device_status(ws), "device status")
    tokens = sample_tokens(T, 16)
    ref, decisive = oracle_block(orc, cfg, W, inp.x_host, inp.bias_host, g, tokens)
    assert decisive.sum() >= len(tokens) - 1, "too many near ties to compare"
    got = out.cpu().numpy()[tokens]
    err = g1_error(got[decisive], ref[decisive])
    assert err.max() <= G1_TOL, (err.max(), err)


@pytest.mark.parametrize("cfg,T,one_launch", [(k3gen.CONFIGS["k3_decode_t8"], 8, False), (SMALL, 40, False),
                                               (k3gen.CONFIGS["k3_decode"], 1, True)])
def test_layer_residual_in_place(cfg, T, one_launch):
    """h_out may be h: the same bf16 bytes as a separate output buffer."""
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    gd = torch.from_numpy(k3gen.norm_weights(cfg).view(np.int16)).cuda()
    dims = dims_of(cfg, m.K3MOE_ONE_LAUNCH if one_launch else 0)
    ws = m.new_workspace(dims, T)
    out = torch.empty((T, cfg.d), dtype=torch.int16, device="cuda")
    m.check(m.k3moe_layer_residual(inp.x, T, gd, EPS, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims,
                                   out, ws), "residual")
    h = inp.x.clone()
    m.check(m.k3moe_layer_residual(h, T, gd, EPS, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims,
                                   h, ws), "residual in place")
    torch.cuda.synchronize()
    assert torch.equal(h, out)
