"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on every
workload shape plus ragged and degenerate cases.  Rules in tests/parity.py."""
import ctypes

import numpy as np
import pytest
import torch

import k3gen
from k3gen import device as kdev
from gpu_helpers import (dims_of, last_group_of_busiest_expert, oracle_reference, run_layer,
                         sample_tokens)
from parity import G1_TOL, check_topk_row, g1_error

pytestmark = pytest.mark.gpu

m = pytest.importorskip("mxfp4_routed_expert_softmax_b200") if torch.cuda.is_available() else None


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    kdev.release_all()


# tokens compared with the oracle per workload; on the grouped-prefill
# workloads the tokens of the busiest expert's last (ragged) group are added
SAMPLES = {"tiny": 4, "k3_decode": 1, "k3_decode_t8": 8, "k3_prefill_512": 64, "k3_prefill_4096": 64}


@pytest.mark.parametrize("name", list(k3gen.CONFIGS))
def test_layer_parity(orc, name):
    cfg = k3gen.CONFIGS[name]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg)
    T = inp.T
    y32, idx, w = run_layer(cfg, W, inp.x, inp.bias, T, m.K3MOE_OUT_FP32)
    y16, idx2, w2 = run_layer(cfg, W, inp.x, inp.bias, T, 0)
    # G2: bf16 output is the RNE rounding of the fp32 result of the same computation
    assert np.array_equal(idx, idx2) and np.array_equal(w, w2)
    r = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(r, y16), "bf16 output is not RNE(fp32 output)"
    tokens = sample_tokens(T, SAMPLES[name])
    if T > 8:
        tail, _, _ = last_group_of_busiest_expert(idx)
        tokens = sorted(set(tokens) | set(tail))
    yo, problems, nd, probs, idx_use, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx,
                                                         tokens)
    assert not problems, problems[:5]
    # routing weights: fp32 softmax vs fp64
    wref = np.take_along_axis(probs, idx[tokens].astype(np.int64), axis=1)
    assert np.allclose(w[tokens], wref, rtol=1e-5, atol=1e-7)
    err = g1_error(y32[tokens], yo)
    assert err.max() <= G1_TOL, (err.max(), err)


def test_route_parity_all_tokens(orc):
    """k3moe_route alone on every token of the 512-token workload."""
    cfg = k3gen.CONFIGS["k3_prefill_512"]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg)
    dims = dims_of(cfg)
    ws = m.new_workspace(dims, inp.T)
    idx = torch.empty((inp.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((inp.T, cfg.k), dtype=torch.float32, device="cuda")
    m.check(m.k3moe_route(inp.x, inp.T, W.w_router, inp.bias, dims, idx, w, ws), "route")
    idx = idx.cpu().numpy()
    w = w.cpu().numpy()
    logits, probs, _, _ = orc.route(inp.x_host, W.w_router_host, inp.bias_host, cfg.k)
    bad = []
    for t in range(inp.T):
        _, pr = check_topk_row(logits[t], idx[t], cfg.k)
        bad += pr
    assert not bad, bad[:5]
    wref = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
    assert np.allclose(w, wref, rtol=1e-5, atol=1e-7)


@pytest.mark.parametrize("name,T", [("tiny", 4), ("tiny", 13), ("k3_decode", 8), ("k3_decode", 3)])
def test_expert_ffn_parity(orc, name, T):
    cfg = k3gen.CONFIGS[name]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    dims = dims_of(cfg, m.K3MOE_OUT_FP32)
    ws = m.new_workspace(dims, T)
    for e in (0, cfg.E // 2, cfg.E - 1):
        out = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
        m.check(m.k3moe_expert_ffn(inp.x, T, W.blobs[e], dims, out, ws), "expert_ffn")
        torch.cuda.synchronize()
        ref = orc.expert_ffn(inp.x_host, W.blob_host(e), cfg.d, cfg.ff)
        err = g1_error(out.cpu().numpy(), ref)
        assert err.max() <= G1_TOL, (e, err)


def test_layer_no_shared_routed_only(orc):
    """The routed sum alone (shared expert off) so the shared term cannot hide
    routed errors."""
    cfg = k3gen.CONFIGS["k3_decode_t8"]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg)
    y, idx, w = run_layer(cfg, W, inp.x, inp.bias, inp.T, m.K3MOE_OUT_FP32 | m.K3MOE_NO_SHARED)
    tokens = list(range(inp.T))
    yo, problems, _, _, _, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx, tokens,
                                             shared=False)
    assert not problems
    assert g1_error(y, yo).max() <= G1_TOL


SMALL = k3gen.Config("small", d=512, ff=256, E=64, k=8, ff_shared=192, T=0, bias="normal")


@pytest.mark.parametrize("T", [1, 5, 8, 9, 17, 30])
def test_ragged_token_counts(orc, T):
    cfg = SMALL
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    y, idx, w = run_layer(cfg, W, inp.x, inp.bias, T, m.K3MOE_OUT_FP32)
    yo, problems, _, _, _, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx,
                                             list(range(T)))
    assert not problems, problems[:3]
    assert g1_error(y, yo).max() <= G1_TOL


@pytest.mark.parametrize("E,k", [(8, 1), (8, 8), (64, 32), (1, 1)])
def test_degenerate_k(orc, E, k):
    cfg = k3gen.Config("deg", d=256, ff=128, E=E, k=k, ff_shared=128, T=0)
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=6)
    y, idx, w = run_layer(cfg, W, inp.x, inp.bias, 6, m.K3MOE_OUT_FP32)
    yo, problems, _, probs, _, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx,
                                                 list(range(6)))
    assert not problems
    if k == E:
        assert np.allclose(w.sum(1), 1.0, rtol=1e-5)
    assert g1_error(y, yo).max() <= G1_TOL


def test_ties_go_to_lower_index(orc):
    """A zero router and zero bias make every logit 0: the selection must be
    experts 0..k-1 in order, each with weight 1/E."""
    cfg = k3gen.Config("ties", d=256, ff=128, E=32, k=4, ff_shared=128, T=0)
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=3)
    zero = torch.zeros_like(W.w_router)
    dims = dims_of(cfg, m.K3MOE_OUT_FP32)
    ws = m.new_workspace(dims, 3)
    idx = torch.empty((3, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((3, cfg.k), dtype=torch.float32, device="cuda")
    m.check(m.k3moe_route(inp.x, 3, zero, None, dims, idx, w, ws), "route")
    assert np.array_equal(idx.cpu().numpy(), np.tile(np.arange(cfg.k), (3, 1)))
    assert np.allclose(w.cpu().numpy(), 1.0 / cfg.E)
    # equal bias on a few experts: ties among them resolve to the lower index
    b = torch.full((cfg.E,), -1.0, device="cuda")
    b[[5, 9, 17, 30, 31]] = 2.0
    m.check(m.k3moe_route(inp.x, 3, zero, b, dims, idx, w, ws), "route")
    assert np.array_equal(idx.cpu().numpy(), np.tile([5, 9, 17, 30], (3, 1)))


def test_deterministic_bytes():
    cfg = k3gen.CONFIGS["k3_decode_t8"]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg)
    a = run_layer(cfg, W, inp.x, inp.bias, inp.T, 0)
    b = run_layer(cfg, W, inp.x, inp.bias, inp.T, 0)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_from_host_matches_device_call():
    cfg = k3gen.CONFIGS["k3_decode_t8"]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg)
    y_dev, _, _ = run_layer(cfg, W, inp.x, inp.bias, inp.T, 0)
    dims = dims_of(cfg)
    ws = m.new_workspace(dims, inp.T, host_staging=True)
    xh = torch.from_numpy(inp.x_host.view(np.int16)).pin_memory()
    yh = torch.empty((inp.T, cfg.d), dtype=torch.int16).pin_memory()
    m.check(m.k3moe_layer_from_host(xh, inp.T, W.w_router, inp.bias, W.blob_ptrs, *W.shared,
                                    dims, yh, ws), "from_host")
    torch.cuda.synchronize()
    assert np.array_equal(yh.numpy(), y_dev)


def test_misaligned_blob_is_reported_not_read():
    cfg = k3gen.CONFIGS["tiny"]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg)
    _, idx, _ = run_layer(cfg, W, inp.x, inp.bias, inp.T, 0)
    bad = W.blob_ptrs.clone()
    bad[int(idx[0, 0])] += 4
    dims = dims_of(cfg)
    ws = m.new_workspace(dims, inp.T)
    y = torch.empty((inp.T, cfg.d), dtype=torch.int16, device="cuda")
    m.check(m.k3moe_layer(inp.x, inp.T, W.w_router, inp.bias, bad, *W.shared, dims, y, None, None,
                          ws), "layer")
    assert m.k3moe_device_status(ws) == m.K3MOE_ERR_DEVICE_CHECK
    # the status is cleared by reading it, and the workspace is usable again
    y2, _, _ = run_layer(cfg, W, inp.x, inp.bias, inp.T, 0)
    assert m.k3moe_device_status(ws) == m.K3MOE_OK


# ----------------------------------------------------------- grouped prefill --
# More than 8 tokens with a workspace sized for them: tokens sorted by expert,
# groups of up to 8 tokens per tensor-core item, expert outputs summed per
# token at the end.  Shapes cover both scale paths (reduction length a
# multiple of 512: scales by TMA; otherwise loaded by the scale warps).

@pytest.mark.parametrize("cfg,T", [
    (k3gen.Config("pf_tiny", d=256, ff=128, E=32, k=4, ff_shared=128, T=0), 64),
    (SMALL, 200),
    (k3gen.Config("pf_k32", d=256, ff=192, E=64, k=32, ff_shared=0, T=0, bias="normal"), 37),
    (k3gen.Config("pf_skew", d=512, ff=512, E=128, k=6, ff_shared=64, T=0, bias="zipf"), 300),
])
def test_grouped_prefill_parity(orc, cfg, T):
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    y32, idx, w = run_layer(cfg, W, inp.x, inp.bias, T, m.K3MOE_OUT_FP32)
    y16, idx2, _ = run_layer(cfg, W, inp.x, inp.bias, T, 0)
    assert np.array_equal(idx, idx2)
    r = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(r, y16), "bf16 output is not RNE(fp32 output)"
    tokens = sample_tokens(T, 24)
    yo, problems, _, probs, _, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx, tokens,
                                                 shared=cfg.ff_shared > 0)
    assert not problems, problems[:3]
    wref = np.take_along_axis(probs, idx[tokens].astype(np.int64), axis=1)
    assert np.allclose(w[tokens], wref, rtol=1e-5, atol=1e-7)
    err = g1_error(y32[tokens], yo)
    assert err.max() <= G1_TOL, (err.max(), err)


def test_grouped_prefill_matches_chunked_path(orc):
    """The same call with a workspace too small for the grouped region runs
    8-token passes; both must meet the oracle, and routing must agree."""
    cfg = SMALL
    T = 45
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    dims = dims_of(cfg, m.K3MOE_OUT_FP32)
    outs = []
    for wsT in (T, 8):
        ws = m.new_workspace(dims, wsT)
        y = torch.empty((T, cfg.d), dtype=torch.float32, device="cuda")
        idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
        m.check(m.k3moe_layer(inp.x, T, W.w_router, inp.bias, W.blob_ptrs, *W.shared, dims, y, idx, w, ws),
                "layer")
        torch.cuda.synchronize()
        m.check(m.k3moe_device_status(ws), "device status")
        outs.append((y.cpu().numpy(), idx.cpu().numpy()))
    assert np.array_equal(outs[0][1], outs[1][1])
    yo, problems, _, _, _, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, outs[0][1],
                                             list(range(T)))
    assert not problems
    for y, _ in outs:
        assert g1_error(y, yo).max() <= G1_TOL


def test_grouped_prefill_deterministic_and_multi_pass(orc):
    """More tokens than one prefill pass takes (8192): two passes; two calls
    give the same bytes."""
    cfg = k3gen.Config("pf_pass", d=256, ff=128, E=64, k=32, ff_shared=128, T=0, bias="normal")
    T = 8192 + 700
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    a = run_layer(cfg, W, inp.x, inp.bias, T, m.K3MOE_OUT_FP32)
    b = run_layer(cfg, W, inp.x, inp.bias, T, m.K3MOE_OUT_FP32)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    y, idx, _ = a
    tokens = sample_tokens(T, 16)
    yo, problems, _, _, _, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx, tokens)
    assert not problems
    assert g1_error(y[tokens], yo).max() <= G1_TOL


@pytest.mark.parametrize("name,T", [("tiny", 1), ("tiny", 4), ("k3_decode", 1), ("k3_decode_t8", 8), ("k3_decode", 3)])
def test_one_launch_parity(orc, name, T):
    """K3MOE_ONE_LAUNCH: the decode pass as one cooperative launch, against the
    oracle on every token, bf16 = RNE(fp32), and against the three launches."""
    cfg = k3gen.CONFIGS[name]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg, T=T)
    one = m.K3MOE_ONE_LAUNCH
    y32, idx, w = run_layer(cfg, W, inp.x, inp.bias, T, m.K3MOE_OUT_FP32 | one, ws_tokens=min(T, 8))
    y16, idx2, w2 = run_layer(cfg, W, inp.x, inp.bias, T, one, ws_tokens=min(T, 8))
    assert np.array_equal(idx, idx2) and np.array_equal(w, w2)
    r = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(r, y16), "bf16 output is not RNE(fp32 output)"
    tokens = list(range(T))
    yo, problems, nd, probs, idx_use, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx, tokens)
    assert not problems, problems[:5]
    wref = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
    assert np.allclose(w, wref, rtol=1e-5, atol=1e-7)
    err = g1_error(y32, yo)
    assert err.max() <= G1_TOL, (err.max(), err)
    # the three-launch pass on the same inputs: same picks, outputs within the gate
    y3, idx3, _ = run_layer(cfg, W, inp.x, inp.bias, T, m.K3MOE_OUT_FP32, ws_tokens=min(T, 8))
    assert np.array_equal(idx, idx3)
    assert g1_error(y3, y32).max() <= G1_TOL
