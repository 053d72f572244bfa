"""The precision of carrying activations as E2M1 pieces (the tensor-core
kernels multiply E2M1 weights by E2M1 activations, so x and w*h enter as a
sum of P pieces, each 32-element block of each piece with its own power-of-two
scale taken from what the earlier pieces left).  A numpy model of that
representation on K3-size matvecs: the G1-style error (per-token max error
over max output) must sit well inside the 2e-3 gate for the piece counts the
kernels use (6 in decode, 4 in the grouped prefill), and each extra piece must
shrink it."""
import numpy as np
import pytest

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def nearest_e2m1(a):
    m = np.abs(a)
    i = np.abs(m[..., None] - E2M1).argmin(-1)
    return np.sign(a) * E2M1[i]


def pieces(v, P):
    """v [..., 32] -> the sum of P pieces (scale 2^e with max|residual| <= 6 * 2^e)."""
    r = v.astype(np.float64).copy()
    out = np.zeros_like(r)
    for _ in range(P):
        amax = np.abs(r).max(-1, keepdims=True)
        e = np.ceil(np.log2(np.maximum(amax, 1e-300) / 6.0))
        q = nearest_e2m1(r / 2.0 ** e) * 2.0 ** e
        q = np.where(amax > 0, q, 0.0)
        out += q
        r -= q
    return out


def g1_like(x, P, W):
    xq = pieces(x.reshape(x.shape[0], -1, 32), P).reshape(x.shape)
    y, yq = x @ W.T, xq @ W.T
    return (np.abs(y - yq).max(1) / np.abs(y).max(1)).max()


@pytest.fixture(scope="module")
def data():
    rng = np.random.default_rng(7)
    d, ff, T = 7168, 1536, 8
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((256, d)) * 0.02          # 256 output rows of a gate/up matrix
    g, u = rng.standard_normal((T, ff)), rng.standard_normal((T, ff))
    h = g / (1 + np.exp(-g)) * u                        # SwiGLU output: heavier tails
    Wd = rng.standard_normal((256, ff)) * 0.02
    return x, W, h, Wd


def test_pieces_keep_the_layer_inside_the_gate(data):
    x, W, h, Wd = data
    for P, bound in ((4, 1e-3), (6, 2e-5)):
        assert g1_like(x, P, W) < bound, P
        assert g1_like(h, P, Wd) < bound, P


def test_each_piece_shrinks_the_error(data):
    x, W, _, _ = data
    errs = [g1_like(x, P, W) for P in (2, 3, 4, 5, 6)]
    assert all(b < a / 4 for a, b in zip(errs, errs[1:])), errs


def test_three_pieces_would_not_do(data):
    """Why not fewer: 3 pieces leave the SwiGLU activations near the gate."""
    _, _, h, Wd = data
    assert g1_like(h, 3, Wd) > 1e-3


def _outliers_every_block(x, rng):
    """One element x2^8 and one x2^10 in every 32-element block."""
    xo = x.copy().reshape(x.shape[0], -1, 32)
    T, nb, _ = xo.shape
    for t in range(T):
        for b in range(nb):
            i, j = rng.choice(32, 2, replace=False)
            xo[t, b, i] *= 2.0 ** 8
            xo[t, b, j] *= 2.0 ** 10
    return xo.reshape(x.shape)


def test_pieces_with_outlier_activations(data):
    """Outliers: a 32-element block whose largest element is 2^10 above the
    others spends its first pieces on that element, so the small ones are
    resolved later; the error is measured against the largest output, which
    the outliers also dominate.  With every block holding a 2^8 and a 2^10
    outlier, or with 8 hidden channels 1000x the others, 4 pieces stay 6x
    inside the 2e-3 gate and 6 pieces ~100x."""
    x, W, h, Wd = data
    rng = np.random.default_rng(11)
    xb = _outliers_every_block(x, rng)
    xc = x.copy()
    xc[:, rng.choice(x.shape[1], 8, replace=False)] *= 1000.0
    hb = _outliers_every_block(h, rng)
    for P, bound in ((4, 3.5e-4 * 1.5), (6, 2e-5)):
        assert g1_like(xb, P, W) < bound, P
        assert g1_like(xc, P, W) < bound, P
        assert g1_like(hb, P, Wd) < bound, P
