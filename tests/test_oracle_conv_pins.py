"""Pins of the oracle's 3x3 convolution and patch matrix (CPU only).

The convolution follows the definition used by deep-learning frameworks for a 3x3 layer
(cross-correlation, stride 1, zero padding 1, no bias).  It is pinned by closed forms
(a centre-only kernel is the identity; a one-hot kernel at (kh, kw) shifts the image by
(kh - 1, kw - 1) with zeros entering at the border), by brute-force Python loops on tiny
inputs, by linearity, and by agreeing with the oracle's sparse product applied to the
oracle's patch matrix.  The patch matrix is pinned against a padded-array slicing
construction.  A planted mistake (a flipped kernel, i.e. true convolution instead of
cross-correlation, or a missing border) must fail the pins.
"""

import numpy as np
import pytest

import oracle


def _tiny(seed, C=3, Nb=2, H=4, W=5, Co=4, density=0.5):
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(C, Nb, H, W))
    Wd = rng.normal(size=(Co, C, 3, 3)) * (rng.random((Co, C, 3, 3)) < density)
    r, c = np.nonzero(Wd.reshape(Co, 9 * C))
    return X, Wd, r.astype(np.int32), c.astype(np.int32), Wd.reshape(Co, 9 * C)[r, c]


def _brute(X, Wd):
    C, Nb, H, W = X.shape
    Co = Wd.shape[0]
    Y = np.zeros((Co, Nb, H, W))
    for co in range(Co):
        for ci in range(C):
            for kh in range(3):
                for kw in range(3):
                    for h in range(H):
                        for w in range(W):
                            hs, ws = h + kh - 1, w + kw - 1
                            if 0 <= hs < H and 0 <= ws < W:
                                Y[co, :, h, w] += Wd[co, ci, kh, kw] * X[ci, :, hs, ws]
    return Y.reshape(Co, -1)


def _shift(X, kh, kw):
    """X shifted so that out[h, w] = X[h + kh - 1, w + kw - 1], zero outside."""
    C, Nb, H, W = X.shape
    P = np.zeros((C, Nb, H + 2, W + 2))
    P[:, :, 1:H + 1, 1:W + 1] = X
    return P[:, :, kh:kh + H, kw:kw + W]


def _patch_by_slicing(X):
    C, Nb, H, W = X.shape
    rows = [_shift(X[ci:ci + 1], k // 3, k % 3).reshape(-1) for ci in range(C) for k in range(9)]
    return np.stack(rows)


@pytest.mark.parametrize("seed", range(4))
def test_conv_matches_brute_force(seed):
    X, Wd, r, c, v = _tiny(seed)
    Y, A = oracle.conv3x3(Wd.shape[0], X.shape[0], X.shape[1], X.shape[2], X.shape[3], r, c, v, X)
    np.testing.assert_allclose(Y, _brute(X, Wd), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(A, _brute(np.abs(X), np.abs(Wd)), rtol=1e-12, atol=1e-12)


def test_conv_centre_is_identity_and_one_hot_is_a_shift():
    X, _, _, _, _ = _tiny(7, C=2, Co=2)
    C, Nb, H, W = X.shape
    for kh in range(3):
        for kw in range(3):
            # output channel co reads input channel co through the tap (kh, kw)
            r = np.arange(C, dtype=np.int32)
            c = (np.arange(C) * 9 + kh * 3 + kw).astype(np.int32)
            Y, _ = oracle.conv3x3(C, C, Nb, H, W, r, c, np.ones(C), X)
            expect = _shift(X, kh, kw).reshape(C, -1)
            assert np.array_equal(Y, expect), (kh, kw)


def test_conv_is_linear_and_equals_product_on_patch_matrix():
    X, Wd, r, c, v = _tiny(3)
    X2 = np.random.default_rng(9).normal(size=X.shape)
    dims = (Wd.shape[0], X.shape[0], X.shape[1], X.shape[2], X.shape[3])
    Y1, _ = oracle.conv3x3(*dims, r, c, v, X)
    Y2, _ = oracle.conv3x3(*dims, r, c, v, X2)
    Y3, _ = oracle.conv3x3(*dims, r, c, v, 2 * X - X2)
    np.testing.assert_allclose(Y3, 2 * Y1 - Y2, rtol=1e-12, atol=1e-12)
    P = oracle.im2col3x3(*dims[1:], X.astype(np.float64))
    Yp, _ = oracle.forward(dims[0], 9 * dims[1], r, c, v, P)
    np.testing.assert_allclose(Yp, Y1, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
def test_patch_matrix_matches_slicing(dtype):
    rng = np.random.default_rng(5)
    X = rng.normal(size=(3, 2, 5, 4)).astype(np.float32)
    if dtype == np.uint16:
        X = (X.view(np.uint32) >> 16).astype(np.uint16)  # any bit patterns will do
    P = oracle.im2col3x3(3, 2, 5, 4, X)
    expect = _patch_by_slicing(X.astype(np.float64)).astype(X.dtype)
    assert P.dtype == X.dtype and P.tobytes() == expect.tobytes()


def test_pins_catch_planted_conv_mistakes():
    X, _, _, _, _ = _tiny(11, C=2, Co=2)
    C, Nb, H, W = X.shape

    def flipped(kh, kw):  # true convolution: taps mirrored
        return _shift(X, 2 - kh, 2 - kw).reshape(C, -1)

    def no_border(kh, kw):  # wrap-around instead of zero padding
        return np.roll(np.roll(X, 1 - kh, axis=2), 1 - kw, axis=3).reshape(C, -1)

    for bad in (flipped, no_border):
        caught = False
        for kh in range(3):
            for kw in range(3):
                if not np.array_equal(bad(kh, kw), _shift(X, kh, kw).reshape(C, -1)):
                    caught = True
        assert caught, bad.__name__
