"""k3moe_layer_noalloc (built-in scratch, no allocation) against k3moe_layer
with a caller workspace: the same bytes, on two calls in a row.  Collected
last, so it runs after every other test has used the library."""
import importlib.util
import os

import numpy as np
import pytest
import torch

import k3gen
from k3gen import device as kdev

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def m():
    spec = importlib.util.spec_from_file_location(
        "k3moe_build", os.path.join(ROOT, "mxfp4_routed_expert_softmax_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import mxfp4_routed_expert_softmax_b200 as m
    return m


def test_noalloc_rejects_shapes_beyond_its_scratch(m):
    """Checked before anything touches the device: no GPU needed."""
    dims = m.make_dims(8192, 3072, 1024, 32, 3072)
    assert m.k3moe_workspace_size(dims, 8) > 16 << 20
    fake = 1 << 20  # never dereferenced: the size check comes first
    st = m.lib.k3moe_layer_noalloc(fake, 1, fake, None, fake, fake, fake, fake, dims, fake, None)
    assert st == m.K3MOE_ERR_WORKSPACE_TOO_SMALL
    assert "16777216" in m.k3moe_last_error()


@pytest.mark.gpu
@pytest.mark.parametrize("name,flags,T", [("tiny", 1, None), ("k3_decode", 0, None),
                                          ("k3_decode_t8", 1, None), ("tiny", 1, 20)])
def test_noalloc_matches_layer_twice(m, name, flags, T):
    """T > 8 runs as 8-token passes on the built-in buffer: the reference is
    k3moe_layer with a workspace sized for 8 tokens (the same passes)."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    cfg = k3gen.CONFIGS[name]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    T = inp.T
    dims = m.make_dims(cfg.d, cfg.ff, cfg.E, cfg.k, cfg.ff_shared, flags)
    out32 = bool(flags & m.K3MOE_OUT_FP32)
    dt = torch.float32 if out32 else torch.int16
    ws = m.new_workspace(dims, min(T, 8))
    y_ref = torch.empty((T, cfg.d), dtype=dt, device="cuda")
    m.check(m.k3moe_layer(inp.x, T, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims, y_ref,
                          None, None, ws), "k3moe_layer")
    torch.cuda.synchronize()
    m.check(m.k3moe_device_status(ws), "device status")
    outs = []
    for _ in range(2):
        y = torch.full((T, cfg.d), -1, dtype=dt, device="cuda")
        m.check(m.k3moe_layer_noalloc(inp.x, T, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims, y),
                "k3moe_layer_noalloc")
        torch.cuda.synchronize()
        outs.append(y.cpu().numpy())
    ref = y_ref.cpu().numpy()
    for o in outs:
        assert np.array_equal(o.view(np.uint8), ref.view(np.uint8))
    kdev.release_all()


@pytest.mark.gpu
def test_noalloc_recovers_after_a_wait_runs_out(m):
    """A call on the built-in buffer whose bounded wait runs out (the failure
    hook, 1 ms bound, no GPU fault) is reported by k3moe_device_status(NULL),
    which also clears the buffer; the next call gives k3moe_layer's bytes."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    cfg = k3gen.CONFIGS["tiny"]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg)
    T = inp.T
    dims = m.make_dims(cfg.d, cfg.ff, cfg.E, cfg.k, cfg.ff_shared, m.K3MOE_OUT_FP32)
    ws = m.new_workspace(dims, T)
    y_ref = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
    m.check(m.k3moe_layer(inp.x, T, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims, y_ref,
                          None, None, ws), "k3moe_layer")
    y = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
    try:
        assert m.k3moe_debug_set_fault(1, 1_000_000) == m.K3MOE_OK
        m.check(m.k3moe_layer_noalloc(inp.x, T, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims, y),
                "k3moe_layer_noalloc")
        torch.cuda.synchronize()
    finally:
        m.k3moe_debug_set_fault(0, 0)
    assert m.k3moe_device_status(None) == m.K3MOE_ERR_DEVICE_TIMEOUT
    assert m.k3moe_device_status(None) == m.K3MOE_OK
    for _ in range(2):
        y.fill_(-1.0)
        m.check(m.k3moe_layer_noalloc(inp.x, T, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims, y),
                "k3moe_layer_noalloc")
        torch.cuda.synchronize()
        assert m.k3moe_device_status(None) == m.K3MOE_OK
        assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32))
    kdev.release_all()
