"""The routing variants on the GPU against the oracle's statement of them:
K3MOE_RENORM_TOPK (the k weights divided by their sum) and
K3MOE_BIAS_SELECT_ONLY (the bias moves the selection, the weights come from
the unbiased softmax), alone and together, on the decode passes and the
grouped path, through k3moe_layer and k3moe_route.  Gates as in parity.py,
with the top-k compared on the selection scores (logit + bias when the bias
moves only the selection)."""
import numpy as np
import pytest
import torch

import k3gen
from gpu_helpers import dims_of, oracle_reference, run_layer, sample_tokens
from k3gen import device as kdev
from parity import G1_TOL, check_topk_row, g1_error

pytestmark = pytest.mark.gpu

m = pytest.importorskip("mxfp4_routed_expert_softmax_b200") if torch.cuda.is_available() else None

SMALL = k3gen.Config("small", d=512, ff=256, E=64, k=8, ff_shared=192, T=0, bias="normal")
TINYB = k3gen.Config("tiny_bias", d=256, ff=128, E=32, k=4, ff_shared=128, T=0, bias="normal")

VARIANTS = [("renorm", True, False), ("select", False, True), ("both", True, True)]


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    kdev.release_all()


def flags_of(renorm, select):
    return (m.K3MOE_RENORM_TOPK if renorm else 0) | (m.K3MOE_BIAS_SELECT_ONLY if select else 0)


@pytest.mark.parametrize("name,renorm,select", VARIANTS)
@pytest.mark.parametrize("cfg,T", [(TINYB, 4), (SMALL, 8), (TINYB, 64), (SMALL, 200),
                                   (k3gen.CONFIGS["k3_decode_t8"], 8)])
def test_layer_routing_variants(orc, cfg, T, name, renorm, select):
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    flags = m.K3MOE_OUT_FP32 | flags_of(renorm, select)
    y, idx, w = run_layer(cfg, W, inp.x, inp.bias, T, flags)
    tokens = sample_tokens(T, 16)
    yo, problems, _, _, _, wref = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx, tokens,
                                                   renorm=renorm, bias_select_only=select)
    assert not problems, problems[:3]
    assert np.allclose(w[tokens], wref, rtol=1e-5, atol=1e-7)
    if renorm:
        assert np.allclose(w.sum(1), 1.0, rtol=1e-5)
    err = g1_error(y[tokens], yo)
    assert err.max() <= G1_TOL, (err.max(), err)


@pytest.mark.parametrize("name,renorm,select", VARIANTS)
def test_route_variants_all_tokens(orc, name, renorm, select):
    """k3moe_route alone, every token of the Zipf-biased 512-token K3 workload
    (the grouped path's router) and of an 8-token pass (decode router)."""
    cfg = k3gen.CONFIGS["k3_prefill_512"]
    W = kdev.weights(cfg)
    for T in (8, 512):
        inp = kdev.DeviceInputs(cfg, T=T)
        dims = dims_of(cfg, flags_of(renorm, select))
        ws = m.new_workspace(dims, T)
        idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
        m.check(m.k3moe_route(inp.x, T, W.w_router, inp.bias, dims, idx, w, ws), "route")
        idx, w = idx.cpu().numpy(), w.cpu().numpy()
        lg, probs, _, _ = orc.route_variant(inp.x_host, W.w_router_host, inp.bias_host, cfg.k,
                                            renorm=renorm, bias_select_only=select)
        scores = lg + inp.bias_host.astype(np.float64) if select else lg
        bad = []
        for t in range(T):
            bad += check_topk_row(scores[t], idx[t], cfg.k)[1]
        assert not bad, bad[:5]
        wref = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
        if renorm:
            wref = wref / wref.sum(1, keepdims=True)
        assert np.allclose(w, wref, rtol=1e-5, atol=1e-7)
