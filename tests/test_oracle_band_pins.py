"""Pins of the oracle's wider-neighbourhood recurrence (CPU only).

oracle.hidden_band links each pixel to the 2r + 1 pixels of the previous line
at orthogonal offsets -r..r, with sigmoid weights normalised over the
neighbours inside the line (CSDN walkthrough "GSPN——在convolution基础上并行序列
建模", section "如何设计一个高效的传播层": the direct method links every pixel to
the whole previous line; r >= K - 1 is that method).  It is pinned to:

* the tridiagonal oracle (itself pinned in test_oracle_pins.py) at r = 1;
* the row-stochastic invariant (theorem 1 of section "方法": a constant line
  stays constant under row-stochastic w);
* closed forms: a single dominant offset shifts the line by that offset every
  step; equal logits at r >= K - 1 average the whole previous line;
* mirror symmetry of the orthogonal axis with reversed offsets;
* restarts of local groups and the stability bound.
"""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(41)


def _first_line_only(shape, d):
    """lambda = 1 on the first line of direction d's scan, 0 elsewhere."""
    lam = np.zeros(shape)
    idx = {0: (..., 0, slice(None)), 1: (..., -1, slice(None)),
           2: (..., slice(None), 0), 3: (..., slice(None), -1)}[d]
    lam[idx] = 1.0
    return lam


@pytest.mark.parametrize("d", [0, 1, 2, 3])
@pytest.mark.parametrize("g", [0, 3])
def test_radius_one_is_the_tridiagonal_layer(d, g):
    x = RNG.normal(size=(2, 2, 7, 9))
    z = RNG.normal(size=(2, 2, 3, 7, 9))
    lam = RNG.uniform(0.2, 1.0, size=(2, 2, 7, 9))
    np.testing.assert_allclose(oracle.hidden_band(x, z, lam, d, 1, g), oracle.hidden(x, z, lam, d, g),
                               rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("d", [0, 1, 2, 3])
@pytest.mark.parametrize("r", [2, 3, 8, 12])
def test_constant_line_stays_constant(d, r):
    H, W = 6, 9
    c = 1.75
    x = np.full((1, 2, H, W), c)
    lam = _first_line_only(x.shape, d)
    z = RNG.normal(scale=3.0, size=(1, 2, 2 * r + 1, H, W))
    h = oracle.hidden_band(x, z, lam, d, r)
    np.testing.assert_allclose(h, c, rtol=1e-13, atol=0)


@pytest.mark.parametrize("o", [-2, -1, 0, 1, 2])
def test_dominant_offset_shifts_the_line(o):
    r, H, W = 2, 6, 20
    x = RNG.normal(size=(1, 1, H, W))
    lam = _first_line_only(x.shape, 0)
    z = np.full((1, 1, 2 * r + 1, H, W), -60.0)
    z[:, :, o + r] = 60.0
    h = oracle.hidden_band(x, z, lam, 0, r)[0, 0]
    for i in range(1, H):
        for k in range(W):
            path = [k + j * o for j in range(i + 1)]
            if all(0 <= q < W for q in path):
                assert abs(h[i, k] - x[0, 0, 0, k + i * o]) < 1e-12, (i, k)


@pytest.mark.parametrize("zval", [-2.0, 0.0, 3.0])
def test_whole_line_band_averages_the_previous_line(zval):
    H, W = 5, 7
    r = W - 1
    x = RNG.normal(size=(1, 1, H, W))
    lam = _first_line_only(x.shape, 0)
    z = np.full((1, 1, 2 * r + 1, H, W), zval)
    h = oracle.hidden_band(x, z, lam, 0, r)[0, 0]
    np.testing.assert_allclose(h[1:], x[0, 0, 0].mean(), rtol=1e-13)


@pytest.mark.parametrize("d", [0, 2])
@pytest.mark.parametrize("r", [1, 2, 4])
def test_mirror_symmetry(d, r):
    H, W = 7, 8
    x = RNG.normal(size=(1, 2, H, W))
    lam = RNG.uniform(0.2, 1.0, size=x.shape)
    z = RNG.normal(size=(1, 2, 2 * r + 1, H, W))
    axis = -1 if d == 0 else -2   # the orthogonal axis of direction d
    h = oracle.hidden_band(x, z, lam, d, r)
    hm = oracle.hidden_band(np.flip(x, axis).copy(), np.flip(np.flip(z, axis), 2).copy(),
                            np.flip(lam, axis).copy(), d, r)
    np.testing.assert_allclose(np.flip(hm, axis), h, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_group_starts_restart(d):
    r, g, H, W = 2, 3, 9, 8
    x = RNG.normal(size=(1, 1, H, W))
    lam = RNG.uniform(0.2, 1.0, size=x.shape)
    z = RNG.normal(size=(1, 1, 2 * r + 1, H, W))
    h = oracle.hidden_band(x, z, lam, d, r, g)[0, 0]
    drive = (lam * x)[0, 0]
    L = H if d < 2 else W
    for c in range(L):
        first = (c % g == 0) if d in (0, 2) else (c % g == g - 1 or c == L - 1)
        if first:
            line = (lambda a: a[c]) if d < 2 else (lambda a: a[:, c])
            np.testing.assert_allclose(line(h), line(drive), rtol=1e-15, atol=1e-15)
    # g = 1: every line restarts
    np.testing.assert_allclose(oracle.hidden_band(x, z, lam, d, r, 1)[0, 0], drive, rtol=1e-15)


def test_stability_bound():
    """Each line is a convex combination of the previous one plus lambda*x,
    so max|h_i| <= max|h_{i-1}| + max|lambda_i x_i|."""
    r, H, W = 3, 12, 10
    x = RNG.normal(scale=5.0, size=(1, 1, H, W))
    lam = RNG.uniform(0.0, 1.0, size=x.shape)
    z = RNG.normal(scale=4.0, size=(1, 1, 2 * r + 1, H, W))
    h = oracle.hidden_band(x, z, lam, 0, r)[0, 0]
    drive = np.abs(lam * x)[0, 0]
    bound = np.abs(h[0]).max()
    for i in range(1, H):
        bound += drive[i].max()
        assert np.abs(h[i]).max() <= bound + 1e-12
