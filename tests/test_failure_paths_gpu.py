"""Device-side failure paths, reached without any GPU fault.

  - K3MOE_STRICT: an E8M0 scale byte of 0xFF (NaN) in a selected expert is
    reported as K3MOE_ERR_DEVICE_CHECK, on the decode and the grouped paths,
    with the weight scales loaded by TMA (K3 shape) and by the scale warps
    (tiny shape); on clean weights the flag changes no output bit.
  - A bounded wait that runs out: the library's failure-path hook makes the
    gate/up pass wait for a signal nobody gives, with a 1 ms bound; the call
    must record K3MOE_ERR_DEVICE_TIMEOUT (nothing faults, the context stays
    usable) and, once the workspace is zero-filled again as the header
    requires, the next call must give the same bytes as before the failure.
"""
import numpy as np
import pytest
import torch

import k3gen
from gpu_helpers import dims_of
from k3gen import device as kdev

pytestmark = pytest.mark.gpu

m = pytest.importorskip("mxfp4_routed_expert_softmax_b200") if torch.cuda.is_available() else None


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    m.k3moe_debug_set_fault(0, 0)
    kdev.release_all()


def call(cfg, W, x, T, flags, ptrs, ws):
    dims = dims_of(cfg, flags)
    y = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    m.check(m.k3moe_layer(x, T, W.w_router, None, ptrs, *W.shared, dims, y, idx, None, ws), "layer")
    return y, idx


def nan_scale_copy(cfg, W, e):
    """Expert e's blob with one W_g scale byte (row 3, block 1) set to 0xFF."""
    blob = W.blob_host(e).copy()
    g_sc = k3gen.plane_offsets(cfg.d, cfg.ff)[1]
    blob[g_sc + 3 * (cfg.d // 32) + 1] = 0xFF
    return torch.from_numpy(blob).cuda()


@pytest.mark.parametrize("name,T", [("tiny", 4), ("tiny", 64), ("k3_decode", 1), ("k3_decode", 40)])
def test_strict_reports_nan_scales(name, T):
    cfg = k3gen.CONFIGS[name]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    base = m.K3MOE_OUT_FP32
    dims = dims_of(cfg, base)
    ws = m.new_workspace(dims, T)
    y0, idx = call(cfg, W, inp.x, T, base, W.blob_ptrs, ws)
    torch.cuda.synchronize()
    assert m.k3moe_device_status(ws) == m.K3MOE_OK
    # strict on clean weights: the same bytes, no report
    y1, _ = call(cfg, W, inp.x, T, base | m.K3MOE_STRICT, W.blob_ptrs, ws)
    torch.cuda.synchronize()
    assert m.k3moe_device_status(ws) == m.K3MOE_OK
    assert torch.equal(y0.view(torch.int32), y1.view(torch.int32))
    # a NaN scale byte in an expert the first token selects
    e = int(idx[0, 0])
    bad = nan_scale_copy(cfg, W, e)
    ptrs = W.blob_ptrs.clone()
    ptrs[e] = bad.data_ptr()
    call(cfg, W, inp.x, T, base | m.K3MOE_STRICT, ptrs, ws)
    torch.cuda.synchronize()
    assert m.k3moe_device_status(ws) == m.K3MOE_ERR_DEVICE_CHECK
    # the report is cleared by reading it; the workspace serves the next call
    y2, _ = call(cfg, W, inp.x, T, base | m.K3MOE_STRICT, W.blob_ptrs, ws)
    torch.cuda.synchronize()
    assert m.k3moe_device_status(ws) == m.K3MOE_OK
    assert torch.equal(y0.view(torch.int32), y2.view(torch.int32))
    del bad


@pytest.mark.parametrize("name,T", [("tiny", 4), ("k3_decode", 1)])
def test_wait_that_runs_out_is_reported_and_recovered(name, T):
    cfg = k3gen.CONFIGS[name]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    dims = dims_of(cfg, m.K3MOE_OUT_FP32)
    ws = m.new_workspace(dims, T)
    y_ref, _ = call(cfg, W, inp.x, T, m.K3MOE_OUT_FP32, W.blob_ptrs, ws)
    torch.cuda.synchronize()
    assert m.k3moe_device_status(ws) == m.K3MOE_OK
    try:
        assert m.k3moe_debug_set_fault(1, 1_000_000) == m.K3MOE_OK  # 1 ms bound
        call(cfg, W, inp.x, T, m.K3MOE_OUT_FP32, W.blob_ptrs, ws)
        torch.cuda.synchronize()
    finally:
        m.k3moe_debug_set_fault(0, 0)
    assert m.k3moe_device_status(ws) == m.K3MOE_ERR_DEVICE_TIMEOUT
    ws.zero_()
    y, _ = call(cfg, W, inp.x, T, m.K3MOE_OUT_FP32, W.blob_ptrs, ws)
    torch.cuda.synchronize()
    assert m.k3moe_device_status(ws) == m.K3MOE_OK
    assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32))
