"""Parity at the edges of the activation-piece representation.

The tensor-core kernels multiply E2M1 weights by activations carried as sums
of E2M1 pieces (6 per element in decode, 4 in the grouped prefill), each
32-element block of each piece with its own E8M0 scale.  The workloads draw
x ~ N(0,1) and E8M0 bytes in 118..124; these tests move every one of those
away from the typical case, on K3 shapes (d=7168, ff=1536), and compare with
the fp64 oracle under the same gates (parity.py):
  - outlier activations: in every 32-element block one element x2^8 and one
    x2^10 of the rest (decode and grouped paths), and a few hidden channels
    x1000;
  - tokens scaled by 2^+40 and 2^-40, and tokens whose blocks sit at the
    bottom of bf16's range (normal and subnormal) beside ordinary blocks,
    which takes the pieces' exponents to their floor of 2^-126;
  - expert E8M0 bytes uniform over 100..150, and single rows at the ends of
    the E8M0 range (bytes 1 and 254).
"""
import numpy as np
import pytest
import torch

import k3gen
from gpu_helpers import (bf16_scale, dims_of, last_group_of_busiest_expert, oracle_reference,
                         run_layer, sample_tokens)
from k3gen import device as kdev
from parity import G1_TOL, g1_error

pytestmark = pytest.mark.gpu

m = pytest.importorskip("mxfp4_routed_expert_softmax_b200") if torch.cuda.is_available() else None

K3 = k3gen.CONFIGS["k3_decode_t8"]  # K3 layer shape, router bias ~ N(0,1)


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    kdev.release_all()


def outlier_blocks(x_bits, seed):
    """Two elements of every 32-element block scaled by 2^8 and 2^10 (the
    positions drawn per block)."""
    T, d = x_bits.shape
    rng = np.random.default_rng(seed)
    mask8 = np.zeros((T, d // 32, 32), dtype=bool)
    mask10 = np.zeros_like(mask8)
    for t in range(T):
        for b in range(d // 32):
            i, j = rng.choice(32, 2, replace=False)
            mask8[t, b, i] = True
            mask10[t, b, j] = True
    x = bf16_scale(x_bits, 8, mask8.reshape(T, d))
    return bf16_scale(x, 10, mask10.reshape(T, d))


def outlier_channels(x_bits, seed, n=8, factor=1000.0):
    """A few hidden channels ~1000x the rest (bf16 rounding of the product)."""
    T, d = x_bits.shape
    rng = np.random.default_rng(seed)
    ch = rng.choice(d, n, replace=False)
    f = (x_bits.astype(np.uint32) << 16).view(np.float32).copy()
    f[:, ch] *= factor
    return (f.view(np.uint32) >> 16).astype(np.uint16)  # truncation: still a valid bf16 input


def check_layer(orc, cfg, W, x_bits, bias_dev, bias_host, flags, tokens=None, ws_tokens=None):
    T = x_bits.shape[0]
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    y, idx, w = run_layer(cfg, W, x, bias_dev, T, m.K3MOE_OUT_FP32 | flags, ws_tokens=ws_tokens)
    assert np.isfinite(y).all()
    if tokens is None:
        tokens = list(range(T))
    shared = not (flags & m.K3MOE_NO_SHARED)
    yo, problems, _, probs, _, _ = oracle_reference(orc, cfg, W, x_bits, bias_host, idx, tokens,
                                                 shared=shared)
    assert not problems, problems[:3]
    wref = np.take_along_axis(probs, idx[tokens].astype(np.int64), axis=1)
    # the routing weights' relative error follows the fp32 error of the logits,
    # bounded by 2^-24 log2(d) sum_j |x_j W_r[e, j]| (large with outliers)
    xa = np.abs(k3gen.bf16_to_f32(x_bits[tokens]).astype(np.float64))
    wa = np.abs(W.w_router_host.astype(np.float64))
    lbound = np.array([(xa[i] @ wa[idx[t]].T).max() for i, t in enumerate(tokens)]) * 2.0 ** -24 * np.log2(cfg.d)
    rtol = np.maximum(1e-5, 4 * lbound)[:, None]
    assert np.all(np.abs(w[tokens] - wref) <= 1e-7 + rtol * np.abs(wref)), (rtol.max(), np.abs(w[tokens] - wref).max())
    err = g1_error(y[tokens], yo)
    assert err.max() <= G1_TOL, (err.max(), err)
    return err, idx


@pytest.mark.parametrize("shared", [True, False])
def test_outlier_blocks_decode(orc, shared):
    """6 pieces (decode passes): every block holds a 2^8 and a 2^10 outlier."""
    W = kdev.weights(K3)
    x = outlier_blocks(k3gen.hidden(K3, T=8), seed=1)
    b = kdev.DeviceInputs(K3, T=1).bias
    check_layer(orc, K3, W, x, b, k3gen.bias(K3), 0 if shared else m.K3MOE_NO_SHARED)


@pytest.mark.parametrize("shared", [True, False])
def test_outlier_blocks_grouped(orc, shared):
    """4 pieces (grouped prefill, 64 tokens): the same outliers."""
    W = kdev.weights(K3)
    x = outlier_blocks(k3gen.hidden(K3, T=64), seed=2)
    b = kdev.DeviceInputs(K3, T=1).bias
    check_layer(orc, K3, W, x, b, k3gen.bias(K3), 0 if shared else m.K3MOE_NO_SHARED,
                tokens=sample_tokens(64, 24))


@pytest.mark.parametrize("T", [8, 40])
def test_outlier_channels(orc, T):
    """A few hidden channels 1000x the others (decode at T=8, grouped at 40)."""
    W = kdev.weights(K3)
    x = outlier_channels(k3gen.hidden(K3, T=T), seed=3)
    b = kdev.DeviceInputs(K3, T=1).bias
    check_layer(orc, K3, W, x, b, k3gen.bias(K3), 0, tokens=sample_tokens(T, 16))


def scaled_tokens(T, seed):
    """Token t of a batch: x2^40 (t % 4 == 0), x2^-40 (t % 4 == 1), a quarter
    of its blocks moved to 2^-126 .. 2^-133 (bf16 normal floor and subnormals)
    (t % 4 == 2), unchanged (t % 4 == 3)."""
    x = k3gen.hidden(K3, T=T)
    out = x.copy()
    rng = np.random.default_rng(seed)
    for t in range(T):
        r = t % 4
        if r == 0:
            out[t] = bf16_scale(x[t:t + 1], 40)[0]
        elif r == 1:
            out[t] = bf16_scale(x[t:t + 1], -40)[0]
        elif r == 2:
            blocks = rng.choice(K3.d // 32, K3.d // 128, replace=False)
            mask = np.zeros(K3.d, dtype=bool)
            for bl in blocks:
                mask[32 * bl:32 * bl + 32] = True
            # |x| ~ 1 -> about 2^-124 (normal), then a second step into the subnormals
            tiny = bf16_scale(x[t:t + 1], -124, mask[None])[0]
            half = mask.copy()
            half[np.nonzero(mask)[0][::2]] = False
            f = (tiny.astype(np.uint32) << 16).view(np.float32)
            f = np.where(half, f * np.float32(2.0 ** -6), f)  # subnormal: exact in fp32, then cut to bf16
            out[t] = (f.view(np.uint32) >> 16).astype(np.uint16)
    return out


@pytest.mark.parametrize("T", [8, 24])
def test_scaled_tokens(orc, T):
    """Tokens at 2^+-40 and with blocks at the floor of bf16's range, on the
    decode path (T=8) and the grouped path (T=24).  The routed and shared
    terms are checked apart (no shared expert) and together."""
    W = kdev.weights(K3)
    x = scaled_tokens(T, seed=4)
    b = kdev.DeviceInputs(K3, T=1).bias
    for flags in (0, m.K3MOE_NO_SHARED):
        check_layer(orc, K3, W, x, b, k3gen.bias(K3), flags)


WIDE = k3gen.Config("k3_e8m0_100_150", d=7168, ff=1536, E=64, k=16, ff_shared=1536, T=0,
                    bias="normal", scale_lo=100, scale_count=51)


@pytest.mark.parametrize("T", [8, 48])
def test_e8m0_wide_range(orc, T):
    """Expert E8M0 bytes uniform over 100..150 (weights from 2^-27 to 2^23
    times the E2M1 value): decode passes (T=8) and the grouped path (T=48)."""
    W = kdev.weights(WIDE)
    inp = kdev.DeviceInputs(WIDE, T=T)
    for flags in (0, m.K3MOE_NO_SHARED):
        check_layer(orc, WIDE, W, inp.x_host, inp.bias, inp.bias_host, flags,
                    tokens=sample_tokens(T, 16))


def test_e8m0_extreme_rows_expert_ffn(orc):
    """One K3-shape expert whose W_u rows 5 and 77 carry E8M0 byte 254 (2^127)
    and whose W_d rows 3 and 900 and W_g row 10 carry byte 1 (2^-126), on
    tokens scaled by 2^-100 so that g, u, h and the output stay inside fp32:
    u on the byte-254 rows is ~2^34, so h there (silu(g) ~ g/2 ~ 2^-103
    times u, either sign) dominates every other h (~2^-205, which fp32
    flushes to zero); the byte-1 rows add ~0."""
    cfg = K3
    d, ff = cfg.d, cfg.ff
    blob = k3gen.expert_blob(cfg, 3).copy()
    g_nib, g_sc, u_nib, u_sc, d_nib, d_sc = k3gen.plane_offsets(d, ff)
    for r in (5, 77):
        blob[u_sc + r * (d // 32): u_sc + (r + 1) * (d // 32)] = 254
    blob[g_sc + 10 * (d // 32): g_sc + 11 * (d // 32)] = 1
    for r in (3, 900):
        blob[d_sc + r * (ff // 32): d_sc + (r + 1) * (ff // 32)] = 1
    T = 4
    x_bits = bf16_scale(k3gen.hidden(cfg, T=T), -100)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    dev_blob = torch.from_numpy(blob).cuda()
    dims = dims_of(cfg, m.K3MOE_OUT_FP32)
    ws = m.new_workspace(dims, T)
    out = torch.empty((T, d), dtype=torch.float32, device="cuda")
    m.check(m.k3moe_expert_ffn(x, T, dev_blob, dims, out, ws), "expert_ffn")
    torch.cuda.synchronize()
    m.check(m.k3moe_device_status(ws), "device status")
    ref = orc.expert_ffn(x_bits, blob, d, ff)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(ref).max() > 0
    err = g1_error(got, ref)
    assert err.max() <= G1_TOL, err


def test_grouped_tail_of_busiest_expert_k3(orc):
    """The Zipf-routed 512-token K3 workload: every token of the busiest
    expert's last group (its ragged tail) plus a seeded sample, routed part
    alone (no shared expert) so the shared term cannot hide a routed error."""
    cfg = k3gen.CONFIGS["k3_prefill_512"]
    W = kdev.weights(cfg)
    inp = kdev.DeviceInputs(cfg)
    y, idx, _ = run_layer(cfg, W, inp.x, inp.bias, inp.T, m.K3MOE_OUT_FP32 | m.K3MOE_NO_SHARED)
    tail, e, n = last_group_of_busiest_expert(idx)
    assert n > 32, "the busiest expert should have more than one group"
    tokens = sorted(set(tail) | set(sample_tokens(inp.T, 16, seed=5)))
    yo, problems, _, _, _, _ = oracle_reference(orc, cfg, W, inp.x_host, inp.bias_host, idx, tokens,
                                             shared=False)
    assert not problems, problems[:3]
    err = g1_error(y[tokens], yo)
    assert err.max() <= G1_TOL, (err.max(), e, n)
