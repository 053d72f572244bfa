"""Pins for the fp64 oracle: each check comes from somewhere other than the
oracle's own code -- hand-worked values (tests/golden/), closed forms,
invariants of the layer, brute force with exact rational arithmetic, and an
independent PyTorch fp64 restatement."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import k3gen
from conftest import read_golden

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- formats --

def test_e2m1_all_codes(orc):
    g = read_golden("e2m1_e8m0.txt")
    assert len(g["e2m1"]) == 16
    for code, val in g["e2m1"]:
        got = orc.e2m1(int(code, 16))
        want = float(val)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got)


def test_e8m0_scales(orc):
    g = read_golden("e2m1_e8m0.txt")
    for e, val in g["e8m0"]:
        got = orc.e8m0(int(e))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float.fromhex(val), (e, got)
    # closed form for every byte
    for e in range(255):
        assert orc.e8m0(e) == 2.0 ** (e - 127)


def test_mxfp4_element_layout(orc):
    g = read_golden("mxfp4_layout.txt")
    m = dict((r[0], int(r[1])) for r in g["matrix"] if len(r) == 2)
    rows, cols = m["rows"], m["cols"]
    nib = np.zeros(rows * cols // 2, np.uint8)
    sc = np.zeros(rows * cols // 32, np.uint8)
    # the [matrix] section carries both the sizes and the byte lists
    for row in g["matrix"]:
        if row[0] == "nib":
            nib[int(row[1])] = int(row[2], 16)
        elif row[0] == "scale":
            sc[int(row[1])] = int(row[2])
    for r, c, v in g["expect"]:
        assert orc.mxfp4_weight(nib, sc, cols, int(r), int(c)) == float(v), (r, c)


def test_bf16_rne_cases(orc):
    one = 1.0
    ulp = 2.0 ** -7
    cases = {
        1.0: 0x3F80,
        -2.0: 0xC000,
        one + ulp / 2: 0x3F80,          # tie -> even (mantissa 0)
        one + 3 * ulp / 2: 0x3F82,      # tie -> even (mantissa 2)
        one + ulp / 2 + 2 ** -20: 0x3F81,  # just above the tie
        0.0: 0x0000,
        3.140625: 0x4049,
    }
    for v, bits in cases.items():
        assert int(orc.bf16_rne(v)) == bits, (v, hex(int(orc.bf16_rne(v))))
    # library second opinion: torch's float32 -> bfloat16 is round-to-nearest-even
    v = RNG.standard_normal(2000).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = orc.bf16_rne(v.astype(np.float64))
    assert np.array_equal(got, ref)


# ---------------------------------------------------------- exact matvec --

E2M1_FRAC = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
             Fraction(4), Fraction(6)]


def _frac_weight(nib, sc, cols, r, c):
    b = int(nib[r * cols // 2 + c // 2])
    code = (b >> 4) if c & 1 else (b & 15)
    v = E2M1_FRAC[code & 7] * (-1 if code & 8 else 1)
    return v * Fraction(2) ** (int(sc[r * cols // 32 + c // 32]) - 127)


def test_mxfp4_matvec_exact_bruteforce(orc):
    """Dyadic inputs make every product and partial sum exact in fp64, so the
    oracle must equal an exact rational computation bit for bit."""
    rows, cols = 5, 96
    nib = RNG.integers(0, 256, rows * cols // 2, dtype=np.uint8)
    sc = RNG.integers(118, 131, rows * cols // 32, dtype=np.uint8)
    xv = RNG.integers(-64, 65, cols) / 16.0
    got = orc.mxfp4_matvec(nib, sc, rows, cols, xv)
    for r in range(rows):
        exact = sum(_frac_weight(nib, sc, cols, r, c) * Fraction(xv[c]) for c in range(cols))
        assert got[r] == float(exact), r


def test_router_logits_exact_bruteforce(orc):
    T, d, E = 3, 64, 7
    xb = RNG.integers(-16, 17, (T, d)) / 8.0
    x = np.array([[k3gen.bf16_bits(v) for v in row] for row in xb], dtype=np.uint16)
    w = (RNG.integers(-32, 33, (E, d)) / 64.0).astype(np.float32)
    b = (RNG.integers(-8, 9, E) / 4.0).astype(np.float32)
    got = orc.router_logits(x, w, b)
    for t in range(T):
        for e in range(E):
            exact = sum(Fraction(xb[t, j]) * Fraction(float(w[e, j])) for j in range(d))
            assert got[t, e] == float(exact + Fraction(float(b[e])))
    # bias = None means no bias
    assert np.array_equal(orc.router_logits(x, w, None) + b.astype(np.float64), got)


# ------------------------------------------------------- softmax / top-k --

def test_softmax_closed_forms(orc):
    for E in (1, 4, 896):
        p = orc.softmax(np.full(E, 0.37))
        assert np.allclose(p, 1.0 / E, rtol=1e-15, atol=0)
    for l1, l2 in [(0.0, 1.0), (2.5, -3.0), (700.0, 699.0), (-800.0, -790.0)]:
        p = orc.softmax(np.array([l1, l2]))
        assert abs(p[0] - 1.0 / (1.0 + math.exp(l2 - l1))) <= 1e-15
    l = RNG.standard_normal(896) * 3
    p = orc.softmax(l)
    assert abs(p.sum() - 1.0) < 1e-14
    # shift invariance, and large logits do not overflow
    assert np.allclose(orc.softmax(l + 500.0), p, rtol=1e-12, atol=0)


def test_topk_bruteforce_random_and_ties(orc):
    for trial in range(50):
        E = int(RNG.integers(1, 300))
        k = int(RNG.integers(1, min(E, 32) + 1))
        if trial % 2:
            l = RNG.integers(-3, 4, E).astype(np.float64)  # heavy ties
        else:
            l = RNG.standard_normal(E)
        want = sorted(range(E), key=lambda e: (-l[e], e))[:k]
        assert list(orc.topk(l, k)) == want


def test_routing_worked_example(orc):
    g = read_golden("routing_worked.txt")
    logits = [float(v) for v in g["logits"][0]]
    probs = [float(v) for v in g["probs"][0]]
    topk = [int(v) for v in g["topk"][0]]
    d, E, k = 32, 4, 2
    x = np.zeros((1, d), np.uint16)
    x[0, 0] = 0x3F80
    w = np.zeros((E, d), np.float32)
    w[:, 0] = logits
    lg, p, idx, wt = orc.route(x, w, None, k)
    assert list(lg[0]) == logits
    assert np.allclose(p[0], probs, rtol=1e-15, atol=0)
    assert list(idx[0]) == topk
    assert np.allclose(wt[0], [probs[i] for i in topk], rtol=1e-15, atol=0)


# ------------------------------------------------------------ expert FFN --

def _golden_expert():
    g = read_golden("expert_ffn_worked.txt")
    sz = dict((a, int(b)) for a, b in g["size"])
    d, ff = sz["d"], sz["ff"]
    offs = k3gen.plane_offsets(d, ff)
    blob = np.zeros(k3gen.blob_bytes(d, ff), np.uint8)
    # unlisted scale bytes are 127 (x1)
    mat = d * ff
    for p in (1, 3, 5):
        blob[offs[p]:offs[p] + mat // 32] = 127
    for plane, i, v in g["bytes"]:
        blob[offs[int(plane)] + int(i)] = int(v, 0)
    x = np.zeros((1, d), np.uint16)
    for j, v in g["x"]:
        x[0, int(j)] = k3gen.bf16_bits(float(v))
    expect = {int(i): float(v) for i, v in g["expect"]}
    return d, ff, x, blob, expect


def test_expert_ffn_worked_example(orc):
    d, ff, x, blob, expect = _golden_expert()
    o = orc.expert_ffn(x, blob, d, ff)[0]
    for i in range(d):
        want = expect.get(i, 0.0)
        if want == 0.0:
            assert o[i] == 0.0, i
        else:
            assert abs(o[i] - want) <= 4e-16 * abs(want), (i, o[i], want)


def _small_cfg(T=3, d=128, ff=64, E=12, k=3, ffs=64, bias=None):
    return k3gen.Config("small", d=d, ff=ff, E=E, k=k, ff_shared=ffs, T=T, bias=bias)


def _inputs(cfg, seed=0):
    x = k3gen.hidden(cfg, seed)
    w = k3gen.router(cfg, seed)
    b = k3gen.bias(cfg, seed)
    blobs = k3gen.all_blobs(cfg, seed)
    sh = k3gen.shared(cfg, seed) if cfg.ff_shared else None
    return x, w, b, blobs, sh


def test_zero_expert_gives_zero(orc):
    cfg = _small_cfg()
    x = k3gen.hidden(cfg)
    blob = k3gen.expert_blob(cfg, 0)
    offs = k3gen.plane_offsets(cfg.d, cfg.ff)
    z = blob.copy()
    for p in (0, 2, 4):  # all-zero nibbles in every matrix
        z[offs[p]:offs[p] + cfg.d * cfg.ff // 2] = 0
    assert np.all(orc.expert_ffn(x, z, cfg.d, cfg.ff) == 0.0)
    # zero W_d alone also gives zero; zero W_u alone makes h = 0
    for p in (2, 4):
        z = blob.copy()
        z[offs[p]:offs[p] + cfg.d * cfg.ff // 2] = 0
        assert np.all(orc.expert_ffn(x, z, cfg.d, cfg.ff) == 0.0)


def test_scale_plus_one_doubles(orc):
    """+1 on every E8M0 byte of W_u (or W_d) doubles the expert output
    exactly (u and h scale by 2, silu(g) is untouched); +1 on W_g does not."""
    cfg = _small_cfg()
    x = k3gen.hidden(cfg)
    blob = k3gen.expert_blob(cfg, 3)
    offs = k3gen.plane_offsets(cfg.d, cfg.ff)
    o = orc.expert_ffn(x, blob, cfg.d, cfg.ff)
    for p in (3, 5):
        b2 = blob.copy()
        b2[offs[p]:offs[p] + cfg.d * cfg.ff // 32] += 1
        assert np.array_equal(orc.expert_ffn(x, b2, cfg.d, cfg.ff), 2.0 * o)
    b2 = blob.copy()
    b2[offs[1]:offs[1] + cfg.d * cfg.ff // 32] += 1
    assert not np.allclose(orc.expert_ffn(x, b2, cfg.d, cfg.ff), 2.0 * o)


def test_negating_up_nibbles_negates_output(orc):
    """Flipping the sign bit of every W_u nibble negates u, h and o."""
    cfg = _small_cfg()
    x = k3gen.hidden(cfg)
    blob = k3gen.expert_blob(cfg, 5)
    offs = k3gen.plane_offsets(cfg.d, cfg.ff)
    b2 = blob.copy()
    b2[offs[2]:offs[2] + cfg.d * cfg.ff // 2] ^= 0x88
    assert np.array_equal(orc.expert_ffn(x, b2, cfg.d, cfg.ff), -orc.expert_ffn(x, blob, cfg.d,
                                                                                 cfg.ff))


# ----------------------------------------------------------------- layer --

def test_layer_k1_no_shared_is_single_expert(orc):
    cfg = _small_cfg(k=1, ffs=0)
    x, w, b, blobs, _ = _inputs(cfg)
    y, idx, wt = orc.layer(x, w, b, blobs, None, cfg.d, cfg.ff, 1)
    _, p, _, _ = orc.route(x, w, b, 1)
    for t in range(cfg.T):
        e = int(idx[t, 0])
        assert e == int(np.argmax(p[t]))
        o = orc.expert_ffn(x[t:t + 1], blobs[e], cfg.d, cfg.ff)[0]
        assert np.array_equal(y[t], p[t, e] * o)


def test_layer_k_equals_E_is_full_mixture(orc):
    cfg = _small_cfg(E=6, k=6, ffs=64)
    x, w, b, blobs, sh = _inputs(cfg)
    y, idx, wt = orc.layer(x, w, b, blobs, sh, cfg.d, cfg.ff, cfg.k)
    _, p, _, _ = orc.route(x, w, b, cfg.k)
    s = orc.shared_ffn(x, *sh)
    mix = s.copy()
    for e in range(cfg.E):
        mix += p[:, e:e + 1] * orc.expert_ffn(x, blobs[e], cfg.d, cfg.ff)
    assert np.allclose(y, mix, rtol=1e-13, atol=1e-13 * np.abs(y).max())
    assert np.allclose(wt.sum(1), 1.0, rtol=1e-14)


def test_layer_relabel_invariance(orc):
    cfg = _small_cfg(bias="normal")
    x, w, b, blobs, sh = _inputs(cfg)
    y, idx, wt = orc.layer(x, w, b, blobs, sh, cfg.d, cfg.ff, cfg.k)
    perm = RNG.permutation(cfg.E)         # new label n holds old expert perm[n]
    inv = np.argsort(perm)
    y2, idx2, wt2 = orc.layer(x, w[perm], b[perm], blobs[perm], sh, cfg.d, cfg.ff, cfg.k)
    # the softmax denominator is summed in a different order, so the weights
    # (and y) agree to rounding, while the selection maps exactly
    assert np.array_equal(inv[idx], idx2)
    assert np.allclose(wt2, wt, rtol=1e-14, atol=0)
    assert np.allclose(y2, y, rtol=1e-13, atol=1e-13 * np.abs(y).max())


def test_layer_shared_only_adds(orc):
    cfg = _small_cfg()
    x, w, b, blobs, sh = _inputs(cfg)
    y, _, _ = orc.layer(x, w, b, blobs, sh, cfg.d, cfg.ff, cfg.k)
    y0, _, _ = orc.layer(x, w, b, blobs, None, cfg.d, cfg.ff, cfg.k)
    s = orc.shared_ffn(x, *sh)
    assert np.allclose(y - y0, s, rtol=1e-12, atol=1e-12 * np.abs(s).max())


def test_bias_shifts_routing(orc):
    cfg = _small_cfg(bias="normal")
    x, w, b, blobs, _ = _inputs(cfg)
    l0 = orc.router_logits(x, w, None)
    lb, p, idx, wt = orc.route(x, w, b, cfg.k)
    assert np.array_equal(lb, l0 + b.astype(np.float64))
    for t in range(cfg.T):
        want = sorted(range(cfg.E), key=lambda e: (-lb[t, e], e))[:cfg.k]
        assert list(idx[t]) == want


# ------------------------------------------------ library second opinion --

def _torch_decode(blob, d, ff):
    """PyTorch fp64 restatement: decode the three matrices by table lookup."""
    tab = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6],
                       dtype=torch.float64)
    b = torch.from_numpy(np.ascontiguousarray(blob))
    offs = k3gen.plane_offsets(d, ff)
    mats = []
    for m, (rows, cols) in enumerate([(ff, d), (ff, d), (d, ff)]):
        nb = b[offs[2 * m]:offs[2 * m] + rows * cols // 2].to(torch.int64)
        codes = torch.stack([nb & 15, nb >> 4], dim=1).reshape(rows, cols)
        sc = b[offs[2 * m + 1]:offs[2 * m + 1] + rows * cols // 32].to(torch.float64)
        scale = torch.pow(2.0, sc - 127).reshape(rows, cols // 32).repeat_interleave(32, dim=1)
        mats.append(tab[codes] * scale)
    return mats


def _torch_layer(x, w, b, blobs, sh, d, ff, k):
    xt = torch.from_numpy(k3gen.bf16_to_f32(x)).to(torch.float64)
    logits = xt @ torch.from_numpy(w).to(torch.float64).T
    if b is not None:
        logits = logits + torch.from_numpy(b).to(torch.float64)
    p = torch.softmax(logits, dim=1)
    E = w.shape[0]
    # stable descending sort: sort ascending on the negated key, stable keeps index order
    order = torch.sort(-logits, dim=1, stable=True).indices[:, :k]
    y = torch.zeros(xt.shape[0], d, dtype=torch.float64)
    if sh is not None:
        wg, wu, wd = (torch.from_numpy(k3gen.bf16_to_f32(a)).to(torch.float64) for a in sh)
        g = xt @ wg.T
        u = xt @ wu.T
        y += (torch.nn.functional.silu(g) * u) @ wd.T
    cache = {}
    for t in range(xt.shape[0]):
        for j in range(k):
            e = int(order[t, j])
            if e not in cache:
                cache[e] = _torch_decode(blobs[e], d, ff)
            Wg, Wu, Wd = cache[e]
            h = torch.nn.functional.silu(Wg @ xt[t]) * (Wu @ xt[t])
            y[t] += p[t, e] * (Wd @ h)
    return y.numpy(), order.numpy(), logits.numpy()


@pytest.mark.parametrize("cfgname", ["tiny", "small_bias"])
def test_torch_fp64_second_opinion(orc, cfgname):
    if cfgname == "tiny":
        cfg = k3gen.CONFIGS["tiny"]
    else:
        cfg = _small_cfg(T=5, d=256, ff=128, E=40, k=6, ffs=128, bias="zipf")
    x, w, b, blobs, sh = _inputs(cfg)
    y, idx, wt = orc.layer(x, w, b, blobs, sh, cfg.d, cfg.ff, cfg.k)
    yt, it, lt = _torch_layer(x, w, b, blobs, sh, cfg.d, cfg.ff, cfg.k)
    assert np.array_equal(idx, it)
    assert np.allclose(y, yt, rtol=1e-12, atol=1e-12 * np.abs(yt).max())


def test_torch_fp64_second_opinion_k3_route_and_one_expert(orc):
    """Full K3 router (896 x 7168) and one full-size expert."""
    cfg = k3gen.CONFIGS["k3_decode_t8"]
    x = k3gen.hidden(cfg)[:2]
    w = k3gen.router(cfg)
    b = k3gen.bias(cfg)
    lg, p, idx, wt = orc.route(x, w, b, cfg.k)
    xt = torch.from_numpy(k3gen.bf16_to_f32(x)).to(torch.float64)
    lt = xt @ torch.from_numpy(w).to(torch.float64).T + torch.from_numpy(b).to(torch.float64)
    assert np.allclose(lg, lt.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(p, torch.softmax(lt, 1).numpy(), rtol=1e-12, atol=0)
    order = torch.sort(-lt, dim=1, stable=True).indices[:, :cfg.k].numpy()
    assert np.array_equal(idx, order)
    e = int(idx[0, 0])
    blob = k3gen.expert_blob(cfg, e)
    o = orc.expert_ffn(x[:1], blob, cfg.d, cfg.ff)[0]
    Wg, Wu, Wd = _torch_decode(blob, cfg.d, cfg.ff)
    h = torch.nn.functional.silu(Wg @ xt[0]) * (Wu @ xt[0])
    ot = (Wd @ h).numpy()
    assert np.allclose(o, ot, rtol=1e-12, atol=1e-12 * np.abs(ot).max())


# ------------------------------------------------------ routing variants --
# The pages' routing adds no bias and weights each pick by its raw softmax
# probability; the library also offers a bias that moves only the selection
# and weights renormalised over the k picks.  Pins: closed forms on a
# hand-built router, and invariants on random ones.

def _variant_case():
    """x = (1, 0), W_r rows (e, 0): logits exactly (0, 1, 2, 3)."""
    x = np.array([[k3gen.bf16_bits(1.0), 0]], dtype=np.uint16)
    w = np.array([[0.0, 0.0], [1.0, 0.0], [2.0, 0.0], [3.0, 0.0]], dtype=np.float32)
    b = np.array([10.0, 0.0, 0.0, -10.0], dtype=np.float32)
    return x, w, b


def test_route_variants_closed_forms(orc):
    x, w, b = _variant_case()
    e = math.e
    # no bias: picks 3, 2; renormalised weights e^3, e^2 over their sum
    _, _, idx, wt = orc.route_variant(x, w, None, 2, renorm=True)
    assert idx[0].tolist() == [3, 2]
    assert np.allclose(wt[0], [e ** 3 / (e ** 3 + e ** 2), e ** 2 / (e ** 3 + e ** 2)], rtol=1e-15, atol=0)
    # bias in the logits (the library's default): s = (10, 1, 2, -7), picks 0, 2
    zs = e ** 10 + e + e ** 2 + e ** -7
    _, _, idx, wt = orc.route_variant(x, w, b, 2)
    assert idx[0].tolist() == [0, 2]
    assert np.allclose(wt[0], [e ** 10 / zs, e ** 2 / zs], rtol=1e-14, atol=0)
    _, _, idx, wt = orc.route_variant(x, w, b, 2, renorm=True)
    assert np.allclose(wt[0], [e ** 10 / (e ** 10 + e ** 2), e ** 2 / (e ** 10 + e ** 2)], rtol=1e-14, atol=0)
    # selection-only bias: the same picks, weights from the unbiased softmax
    z = 1 + e + e ** 2 + e ** 3
    lg, _, idx, wt = orc.route_variant(x, w, b, 2, bias_select_only=True)
    assert idx[0].tolist() == [0, 2]
    assert np.array_equal(lg[0], [0.0, 1.0, 2.0, 3.0])
    assert np.allclose(wt[0], [1 / z, e ** 2 / z], rtol=1e-15, atol=0)
    _, _, idx, wt = orc.route_variant(x, w, b, 2, renorm=True, bias_select_only=True)
    assert idx[0].tolist() == [0, 2]
    assert np.allclose(wt[0], [1 / (1 + e ** 2), e ** 2 / (1 + e ** 2)], rtol=1e-15, atol=0)


def test_route_variants_selection_ties_go_to_lower_index(orc):
    """Selection scores tied by the bias: (0+2, 1+1, 2+0, 3-1) all equal 2."""
    x, w, _ = _variant_case()
    b = np.array([2.0, 1.0, 0.0, -1.0], dtype=np.float32)
    _, _, idx, _ = orc.route_variant(x, w, b, 3, bias_select_only=True)
    assert idx[0].tolist() == [0, 1, 2]


def test_route_variants_invariants(orc):
    rng = np.random.default_rng(21)
    T, d, E, k = 5, 64, 40, 6
    x = np.array([[k3gen.bf16_bits(v) for v in row] for row in rng.standard_normal((T, d))],
                 dtype=np.uint16)
    w = (rng.standard_normal((E, d)) / 8).astype(np.float32)
    b = rng.standard_normal(E).astype(np.float32)
    # plain variant = the pages' routing
    l0, p0, i0, w0 = orc.route(x, w, b, k)
    l1, p1, i1, w1 = orc.route_variant(x, w, b, k)
    assert np.array_equal(i0, i1) and np.array_equal(w0, w1) and np.array_equal(l0, l1)
    # renormalised: same picks, weights proportional to p, summing to one
    _, _, i2, w2 = orc.route_variant(x, w, b, k, renorm=True)
    assert np.array_equal(i2, i0)
    assert np.allclose(w2.sum(1), 1.0, rtol=0, atol=1e-15)
    assert np.allclose(w2 / w2[:, :1], w0 / w0[:, :1], rtol=1e-14)
    # k = E: renormalising changes nothing (the probabilities already sum to one)
    _, _, _, wa = orc.route_variant(x, w, b, E)
    _, _, _, wb = orc.route_variant(x, w, b, E, renorm=True)
    assert np.allclose(wa, wb, rtol=1e-14, atol=0)
    # selection-only bias with a zero bias, or none, is the unbiased routing
    l3, _, i3, w3 = orc.route_variant(x, w, np.zeros(E, np.float32), k, bias_select_only=True)
    l4, _, i4, w4 = orc.route(x, w, None, k)
    assert np.array_equal(i3, i4) and np.array_equal(w3, w4) and np.array_equal(l3, l4)
    # selection-only: picks = top-k of (l + b); weights = the unbiased softmax at the picks
    l5, p5, i5, w5 = orc.route_variant(x, w, b, k, bias_select_only=True)
    s = l5 + b.astype(np.float64)
    for t in range(T):
        assert i5[t].tolist() == sorted(range(E), key=lambda e: (-s[t, e], e))[:k]
    unb = np.exp(l5 - l5.max(1, keepdims=True))
    unb /= unb.sum(1, keepdims=True)
    assert np.allclose(w5, np.take_along_axis(unb, i5.astype(np.int64), 1), rtol=1e-13)


# --------------------------------------------- RMSNorm and the residual add --

def _bf16_row(vals):
    return np.array([[k3gen.bf16_bits(v) for v in vals]], dtype=np.uint16)


def test_rmsnorm_worked_example(orc):
    """h = (3, 4), g = (1, 0.5), eps = 0: mean h^2 = 12.5, so x = (3, 2) / sqrt(12.5)
    rounded to bf16 (the generator's own nearest-even rounding)."""
    h = _bf16_row([3.0, 4.0])
    g = np.array([k3gen.bf16_bits(1.0), k3gen.bf16_bits(0.5)], dtype=np.uint16)
    x = orc.rmsnorm(h, g, 0.0)
    r = 1.0 / math.sqrt(12.5)
    assert x[0].tolist() == [k3gen.bf16_bits(3.0 * r), k3gen.bf16_bits(2.0 * r)]


def test_rmsnorm_constant_token_gives_the_weights(orc):
    """h_j = c for all j, eps = 0: x_j = sign(c) g_j exactly."""
    rng = np.random.default_rng(3)
    g = np.array([k3gen.bf16_bits(v) for v in rng.standard_normal(64)], dtype=np.uint16)
    for c in (0.75, -3.0, 1024.0):
        x = orc.rmsnorm(_bf16_row([c] * 64), g, 0.0)
        want = g if c > 0 else (g ^ 0x8000)
        assert np.array_equal(x[0], want)


def test_rmsnorm_scale_invariance_and_eps(orc):
    """Scaling a token by a power of two leaves its norm unchanged (eps = 0);
    eps pulls a small token towards zero."""
    rng = np.random.default_rng(4)
    h = np.array([[k3gen.bf16_bits(v) for v in rng.standard_normal(128)]], dtype=np.uint16)
    g = np.array([k3gen.bf16_bits(v) for v in 1 + 0.1 * rng.standard_normal(128)], dtype=np.uint16)
    hf = k3gen.bf16_to_f32(h).astype(np.float64)
    h8 = np.array([[k3gen.bf16_bits(v) for v in hf[0] * 8.0]], dtype=np.uint16)
    assert np.array_equal(orc.rmsnorm(h, g, 0.0), orc.rmsnorm(h8, g, 0.0))
    small = np.array([[k3gen.bf16_bits(v) for v in hf[0] * 1e-3]], dtype=np.uint16)
    a = k3gen.bf16_to_f32(orc.rmsnorm(small, g, 0.0)).astype(np.float64)
    b = k3gen.bf16_to_f32(orc.rmsnorm(small, g, 1e-4)).astype(np.float64)
    ms = (hf[0] * 1e-3) ** 2
    assert np.allclose(b / a, math.sqrt(ms.mean() / (ms.mean() + 1e-4)), rtol=2e-2)


def test_residual_add(orc):
    h = _bf16_row([1.5, -2.0, 0.25])
    y = np.array([[0.125, 4.0, -0.25]])
    assert np.array_equal(orc.residual_add(h, y), [[1.625, 2.0, 0.0]])
