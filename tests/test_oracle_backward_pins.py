"""Pins of the oracle's backward pass (CPU only).

The backward is the gradient of L = sum(gy * y) with respect to x, the
logits, lambda and u.  It is pinned to the forward oracle (itself pinned to
the pages in test_oracle_pins.py) by central finite differences on tiny
planes, and by closed forms: du_d = gy * h_d, and logits of a one-wide line
have no effect (their gradient is zero).
"""
import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(7)


def _rand_inputs(B, C, H, W, logit_std=1.0):
    x = RNG.normal(size=(B, C, H, W))
    z = [RNG.normal(scale=logit_std, size=(B, C, 3, H, W)) for _ in range(4)]
    lam = [RNG.uniform(0.2, 1.0, size=(B, C, H, W)) for _ in range(4)]
    u = [RNG.normal(size=(B, C, H, W)) for _ in range(4)]
    gy = RNG.normal(size=(B, C, H, W))
    return x, z, lam, u, gy


def _loss(x, z, lam, u, gy, g):
    return float(np.sum(gy * oracle.forward(x, z, lam, u, g)))


def _fd_check(arr, grad, f, eps=1e-6, tol=1e-6):
    """Central differences of f() with respect to every entry of arr."""
    flat = arr.reshape(-1)
    num = np.empty(flat.size)
    for j in range(flat.size):
        keep = flat[j]
        flat[j] = keep + eps
        fp = f()
        flat[j] = keep - eps
        fm = f()
        flat[j] = keep
        num[j] = (fp - fm) / (2 * eps)
    scale = max(np.abs(num).max(), 1e-12)
    err = np.abs(num - grad.reshape(-1)).max() / scale
    assert err <= tol, f"finite-difference mismatch {err:.2e}"


@pytest.mark.parametrize("H,W,g", [(3, 4, 0), (4, 3, 0), (5, 4, 2), (4, 5, 3), (1, 5, 0),
                                   (5, 1, 0)])
def test_backward_matches_finite_differences(H, W, g):
    x, z, lam, u, gy = _rand_inputs(1, 2, H, W)
    dx, dz, dl, du = oracle.backward(x, z, lam, u, gy, g)
    f = lambda: _loss(x, z, lam, u, gy, g)
    _fd_check(x, dx, f)
    for d in range(4):
        _fd_check(z[d], dz[d], f)
        _fd_check(lam[d], dl[d], f)
        _fd_check(u[d], du[d], f)


def test_du_is_gy_times_hidden_state():
    x, z, lam, u, gy = _rand_inputs(2, 3, 6, 7)
    _, _, _, du = oracle.backward(x, z, lam, u, gy, 0)
    for d in range(4):
        h = oracle.hidden(x, z[d], lam[d], d, 0)
        np.testing.assert_allclose(du[d], gy * h, rtol=1e-13, atol=1e-13)


def test_one_wide_lines_have_no_logit_gradient():
    """A one-column plane scanned vertically (and a one-row plane scanned
    horizontally) has one pixel per line: its single weight is 1 whatever
    the logits, so their gradient is exactly zero."""
    x, z, lam, u, gy = _rand_inputs(1, 2, 6, 1)
    _, dz, _, _ = oracle.backward(x, z, lam, u, gy, 0)
    assert np.all(dz[0] == 0) and np.all(dz[1] == 0)
    x, z, lam, u, gy = _rand_inputs(1, 2, 1, 6)
    _, dz, _, _ = oracle.backward(x, z, lam, u, gy, 0)
    assert np.all(dz[2] == 0) and np.all(dz[3] == 0)


def test_group_len_one_makes_logits_irrelevant():
    x, z, lam, u, gy = _rand_inputs(1, 2, 5, 6)
    dx, dz, dl, _ = oracle.backward(x, z, lam, u, gy, 1)
    for d in range(4):
        assert np.all(dz[d] == 0)
        np.testing.assert_allclose(dl[d], x * u[d] * gy, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dx, sum(lam[d] * u[d] for d in range(4)) * gy, rtol=1e-12)


def test_backward_is_linear_in_gy():
    x, z, lam, u, gy = _rand_inputs(1, 3, 5, 5)
    a = oracle.backward(x, z, lam, u, gy, 0)
    b = oracle.backward(x, z, lam, u, 2.5 * gy, 0)
    np.testing.assert_allclose(b[0], 2.5 * a[0], rtol=1e-12)
    for d in range(4):
        np.testing.assert_allclose(b[1][d], 2.5 * a[1][d], rtol=1e-12, atol=1e-15)
