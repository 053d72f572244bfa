"""The seeded input generator: published SplitMix64 outputs, determinism,
distributions and layouts."""
import hashlib

import numpy as np

import k3gen

MASK = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def _splitmix64_next(state):
    """SplitMix64 as published (Steele, Lea, Flood 2014 / Vigna's splitmix64.c)."""
    state = (state + GAMMA) & MASK
    z = state
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return state, z ^ (z >> 31)


def test_splitmix64_known_first_output():
    # The first output of SplitMix64 seeded with state 0 is the widely quoted
    # constant 0xE220A8397B1DCDAF.
    _, z = _splitmix64_next(0)
    assert z == 0xE220A8397B1DCDAF


def test_draws_follow_splitmix64_sequence():
    lib = k3gen._load()
    for seed, stream in [(0, 0), (7, 3), (2**40 + 1, 6)]:
        state = lib.k3gen_base(seed, stream)
        for i in range(20):
            state, z = _splitmix64_next(state)
            assert lib.k3gen_draw(seed, stream, i) == z


def _sha(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def test_determinism_and_seed_dependence():
    cfg = k3gen.CONFIGS["tiny"]
    a = [k3gen.hidden(cfg), k3gen.router(cfg), k3gen.all_blobs(cfg)]
    b = [k3gen.hidden(cfg), k3gen.router(cfg), k3gen.all_blobs(cfg)]
    c = [k3gen.hidden(cfg, seed=1), k3gen.router(cfg, seed=1), k3gen.all_blobs(cfg, seed=1)]
    for u, v, w in zip(a, b, c):
        assert _sha(u) == _sha(v)
        assert _sha(u) != _sha(w)


def test_distributions():
    n = 200000
    z = k3gen.normal(0, 0, 0, 2000)
    lib = k3gen._load()
    out = np.empty(n, np.float32)
    lib.k3gen_normal_f32(0, 1, 0, n, 1.0, out.ctypes.data)
    assert abs(out.mean()) < 0.01 and abs(out.std() - 1.0) < 0.01
    assert abs(z.mean()) < 0.1
    cfg = k3gen.CONFIGS["tiny"]
    blob = k3gen.expert_blob(cfg, 0)
    offs = k3gen.plane_offsets(cfg.d, cfg.ff)
    sc = blob[offs[1]:offs[2]]
    assert sc.min() == 118 and sc.max() == 124
    nib = blob[offs[0]:offs[1]]
    lo, hi = nib & 15, nib >> 4
    assert set(np.unique(lo)) == set(range(16)) and set(np.unique(hi)) == set(range(16))
    x = k3gen.bf16_to_f32(k3gen.hidden(cfg))
    assert np.all(np.isfinite(x))


def test_zipf_bias_is_ranked():
    cfg = k3gen.CONFIGS["k3_prefill_512"]
    b = k3gen.bias(cfg)
    r = np.exp(-b.astype(np.float64) / 1.1)
    assert np.allclose(np.sort(r), np.arange(1, cfg.E + 1), rtol=1e-5)


def test_bf16_bits_round_to_nearest_even():
    assert k3gen.bf16_bits(1.0) == 0x3F80
    assert k3gen.bf16_bits(1.0 + 2**-8) == 0x3F80
    assert k3gen.bf16_bits(1.0 + 3 * 2**-8) == 0x3F82
    assert k3gen.bf16_bits(-0.5) == 0xBF00


def test_blob_layout_sizes():
    for cfg in k3gen.CONFIGS.values():
        offs = k3gen.plane_offsets(cfg.d, cfg.ff)
        assert offs[1] - offs[0] == cfg.d * cfg.ff // 2
        assert cfg.blob_bytes == 3 * cfg.d * cfg.ff * 17 // 32
        for o in offs:
            assert o % 16 == 0
    assert k3gen.CONFIGS["k3_decode"].blob_bytes == 17547264


def test_norm_weights_stream():
    """RMSNorm weights: bf16(1 + 0.1 N(0,1)) from stream 7, deterministic."""
    cfg = k3gen.CONFIGS["tiny"]
    g = k3gen.norm_weights(cfg)
    assert g.dtype == np.uint16 and g.shape == (cfg.d,)
    assert np.array_equal(g, k3gen.norm_weights(cfg))
    v = k3gen.bf16_to_f32(g).astype(np.float64)
    assert abs(v.mean() - 1.0) < 0.03 and 0.07 < v.std() < 0.13
    n = k3gen.normal(0, k3gen.STREAM_NORM, 0, 4)
    assert [int(b) for b in g[:4]] == [k3gen.bf16_bits(1.0 + 0.1 * z) for z in n]
