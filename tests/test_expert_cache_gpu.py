"""The expert cache on the GPU: a decode sequence run with only S of the E
experts in device memory (the rest copied in from page-locked host memory as
the routing asks for them) gives the same bytes as the same calls with every
expert resident -- the cache moves bytes, it changes no arithmetic -- and its
counters add up."""
import numpy as np
import pytest
import torch

import k3gen
from gpu_helpers import dims_of
from k3gen import device as kdev

pytestmark = pytest.mark.gpu

m = pytest.importorskip("mxfp4_routed_expert_softmax_b200") if torch.cuda.is_available() else None

K3S = k3gen.Config("k3_e48", d=7168, ff=1536, E=48, k=16, ff_shared=1536, T=0, bias="normal")


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    kdev.release_all()


@pytest.mark.parametrize("cfg,S,T,steps", [(k3gen.Config("tiny_b", d=256, ff=128, E=32, k=4, ff_shared=128, T=0,
                                                         bias="normal"), 8, 2, 16),
                                           (K3S, 24, 1, 6)])
def test_cached_layer_matches_resident(cfg, S, T, steps):
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T * steps)
    dims = dims_of(cfg, m.K3MOE_OUT_FP32)
    host = torch.empty((cfg.E, cfg.blob_bytes), dtype=torch.uint8).pin_memory()
    for e in range(cfg.E):
        host[e].copy_(torch.from_numpy(W.blob_host(e)))
    sb = m.k3moe_cache_slot_bytes(dims)
    slots = torch.empty(S * sb, dtype=torch.uint8, device="cuda")
    table = torch.zeros(cfg.E, dtype=torch.int64, device="cuda")
    cache = m.ExpertCache(dims, S, slots, [host.data_ptr() + e * cfg.blob_bytes for e in range(cfg.E)])
    idx_host = torch.empty(T * cfg.k, dtype=torch.int32).pin_memory()
    ws = m.new_workspace(dims, 8)
    ws_ref = m.new_workspace(dims, 8)
    y = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
    y_ref = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
    idx_ref = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    distinct = 0
    for i in range(steps):
        x = inp.x[i * T:(i + 1) * T].contiguous()
        m.check(m.k3moe_layer_cached(cache, x, T, W.w_router, inp.bias, table, *W.shared, dims, y, idx_host, ws),
                "k3moe_layer_cached")
        m.check(m.k3moe_layer(x, T, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims, y_ref, idx_ref, None,
                              ws_ref), "k3moe_layer")
        torch.cuda.synchronize()
        assert m.k3moe_device_status(ws) == m.K3MOE_OK
        assert np.array_equal(idx_host.numpy().reshape(T, cfg.k), idx_ref.cpu().numpy())
        assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32)), f"step {i}"
        distinct += len(set(idx_host.numpy().tolist()))
    s = cache.stats()
    assert s["requests"] == distinct
    assert s["hits"] + s["fills"] == s["requests"]
    assert s["fills"] >= min(S, distinct) and s["hits"] > 0
    cache.close()
