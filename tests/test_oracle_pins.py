"""Pins of the fp64 CPU oracle against what the GSPN pages and the mathematics fix.

Each test is chosen so that a plausible mistake in the oracle (a dropped
lambda, a sign flip in the sigmoid, a swapped logit slot, a transposed
direction, a wrong border normalisation, an off-by-one in the scan or in the
local groups) fails at least one of them.  Sources are the CSDN walkthrough
"GSPN——在convolution基础上并行序列建模": section "方法" (recurrence, output
gate, unrolled G), "稳定性-上下文条件" (Theorems 1 and 2), "行随机矩阵"
(sigmoid + per-row normalisation), "全局与局部GSPN" (local groups).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import dense_g

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng_global = np.random.default_rng(1234)


def rand_inputs(B, C, H, W, rng, logit_std=1.0):
    x = rng.normal(size=(B, C, H, W))
    z = [rng.normal(scale=logit_std, size=(B, C, 3, H, W)) for _ in range(4)]
    lam = [rng.uniform(size=(B, C, H, W)) for _ in range(4)]
    u = [rng.normal(size=(B, C, H, W)) for _ in range(4)]
    return x, z, lam, u


def scan_lines(d, H, W):
    """Index arrays selecting scan line i (ordered by orthogonal index)."""
    L = H if d < 2 else W
    out = []
    for i in range(L):
        if d == 0:
            out.append((np.full(W, i), np.arange(W)))
        elif d == 1:
            out.append((np.full(W, H - 1 - i), np.arange(W)))
        elif d == 2:
            out.append((np.arange(H), np.full(H, i)))
        else:
            out.append((np.arange(H), np.full(H, W - 1 - i)))
    return out


# --------------------------------------------------------------------------
# Hand-computed example (tests/golden/hand_3x3_top_to_bottom.json)
# --------------------------------------------------------------------------
def _load_hand():
    with open(os.path.join(GOLDEN, "hand_3x3_top_to_bottom.json")) as f:
        g = json.load(f)
    ln3 = g["ln3"]

    def val(v):
        if v == "ln3":
            return ln3
        if v == "-ln3":
            return -ln3
        return float(v)

    x = np.array(g["x"], dtype=np.float64)[None, None]
    lam0 = np.array(g["lam"], dtype=np.float64)[None, None]
    slots = g["wlogit_slots"]
    z0 = np.stack([np.array([[val(v) for v in row] for row in slots[k]])
                   for k in ("slot0_offset_minus1", "slot1_offset_0", "slot2_offset_plus1")])[None, None]
    exp_g = np.array([[float(Fraction(v)) for v in row] for row in g["expected_h_global"]])
    exp_l = np.array([[float(Fraction(v)) for v in row] for row in g["expected_h_group_len_2"]])
    return x, z0, lam0, exp_g, exp_l


def test_hand_example_hidden_global():
    x, z0, lam0, exp_g, _ = _load_hand()
    h = oracle.hidden(x, z0, lam0, d=0, group_len=0)
    np.testing.assert_allclose(h[0, 0], exp_g, rtol=0, atol=1e-13)


def test_hand_example_hidden_local():
    x, z0, lam0, _, exp_l = _load_hand()
    h = oracle.hidden(x, z0, lam0, d=0, group_len=2)
    np.testing.assert_allclose(h[0, 0], exp_l, rtol=0, atol=1e-13)


def test_hand_example_forward_merges_with_u():
    x, z0, lam0, exp_g, _ = _load_hand()
    zeros = np.zeros_like(x)
    rng = np.random.default_rng(5)
    z = [z0] + [rng.normal(size=z0.shape) for _ in range(3)]
    lam = [lam0] + [rng.uniform(size=x.shape) for _ in range(3)]
    u = [np.ones_like(x), zeros, zeros, zeros]
    y = oracle.forward(x, z, lam, u)
    np.testing.assert_allclose(y[0, 0], exp_g, rtol=0, atol=1e-13)
    u2 = [2.5 * np.ones_like(x), zeros, zeros, zeros]
    np.testing.assert_allclose(oracle.forward(x, z, lam, u2)[0, 0], 2.5 * exp_g, atol=1e-12)


# --------------------------------------------------------------------------
# Unrolled lower-triangular G (section "方法")
# --------------------------------------------------------------------------
@pytest.mark.parametrize("H,W", [(1, 1), (1, 4), (4, 1), (2, 3), (3, 5), (5, 4), (6, 6)])
@pytest.mark.parametrize("group_len", [0, 2, 3])
def test_recurrence_equals_unrolled_G(H, W, group_len):
    rng = np.random.default_rng(H * 100 + W * 10 + group_len)
    x, z, lam, _ = rand_inputs(1, 2, H, W, rng, logit_std=1.5)
    for d in range(4):
        h = oracle.hidden(x, z[d], lam[d], d=d, group_len=group_len)
        for c in range(2):
            ref = dense_g.dense_hidden_plane(x[0, c], z[d][0, c], lam[d][0, c], d, group_len)
            np.testing.assert_allclose(h[0, c], ref, rtol=0, atol=1e-12)


def test_forward_equals_dense_forward():
    rng = np.random.default_rng(7)
    x, z, lam, u = rand_inputs(2, 1, 4, 5, rng)
    for g in (0, 2):
        np.testing.assert_allclose(oracle.forward(x, z, lam, u, g),
                                   dense_g.dense_forward(x, z, lam, u, g), atol=1e-12)


def test_forward_is_sum_of_gated_directions():
    rng = np.random.default_rng(8)
    x, z, lam, u = rand_inputs(2, 3, 7, 5, rng)
    y = oracle.forward(x, z, lam, u, 0)
    ref = sum(u[d] * oracle.hidden(x, z[d], lam[d], d) for d in range(4))
    np.testing.assert_allclose(y, ref, atol=1e-12)


# --------------------------------------------------------------------------
# Row-stochastic weights (section "行随机矩阵")
# --------------------------------------------------------------------------
@pytest.mark.parametrize("H,W", [(1, 1), (3, 1), (1, 3), (4, 6)])
def test_weights_row_stochastic_with_border_drop(H, W):
    rng = np.random.default_rng(11)
    z = rng.normal(scale=3.0, size=(1, 1, 3, H, W))
    for d in range(4):
        w = oracle.weights(z, d)[0, 0]
        assert np.all(w >= 0)
        np.testing.assert_allclose(w.sum(axis=0), 1.0, atol=1e-14)
        K = W if d < 2 else H
        # orthogonal coordinate of every pixel
        k = np.broadcast_to(np.arange(W)[None, :], (H, W)) if d < 2 else \
            np.broadcast_to(np.arange(H)[:, None], (H, W))
        assert np.all(w[0][k == 0] == 0.0)              # no left/upper neighbour
        assert np.all(w[2][k == K - 1] == 0.0)          # no right/lower neighbour
        if K == 1:
            np.testing.assert_array_equal(w[1], 1.0)
        else:
            nz = (w > 0).sum(axis=0)
            assert np.all(nz[(k == 0) | (k == K - 1)] == 2)
            assert np.all(nz[(k > 0) & (k < K - 1)] == 3)


def test_weights_match_sigmoid_ratio():
    rng = np.random.default_rng(12)
    z = rng.normal(size=(1, 1, 3, 4, 4))
    w = oracle.weights(z, 0)[0, 0]
    s = 1 / (1 + np.exp(-z[0, 0]))
    r, c = 2, 1  # interior for d=0 (orthogonal = column)
    np.testing.assert_allclose(w[:, r, c], s[:, r, c] / s[:, r, c].sum(), atol=1e-15)


# --------------------------------------------------------------------------
# Theorem 1: row-stochastic products => a constant first line propagates
# unchanged (section "稳定性-上下文条件")
# --------------------------------------------------------------------------
@pytest.mark.parametrize("H,W", [(9, 7), (5, 1), (1, 6), (12, 12)])
def test_constant_first_line_propagates(H, W):
    rng = np.random.default_rng(13)
    for d in range(4):
        x = rng.normal(size=(1, 2, H, W))
        z = rng.normal(scale=2.0, size=(1, 2, 3, H, W))
        lam = np.zeros((1, 2, H, W))
        first = scan_lines(d, H, W)[0]
        lam[0, :, first[0], first[1]] = 1.0
        cst = np.array([1.75, -0.5])
        for c in range(2):
            x[0, c, first[0], first[1]] = cst[c]
        h = oracle.hidden(x, z, lam, d)
        for c in range(2):
            np.testing.assert_allclose(h[0, c], cst[c], atol=1e-12)


def test_constant_propagates_within_each_local_group():
    rng = np.random.default_rng(14)
    H, W, g = 10, 9, 4
    for d in range(4):
        x = rng.normal(size=(1, 1, H, W))
        z = rng.normal(size=(1, 1, 3, H, W))
        lam = np.zeros((1, 1, H, W))
        lines = scan_lines(d, H, W)
        expected = np.zeros((H, W))
        level = 0.0
        for i, (rr, cc) in enumerate(lines):
            if dense_g.group_id(d, H, W, i, g) != (dense_g.group_id(d, H, W, i - 1, g) if i else -1):
                level = rng.normal()
                lam[0, 0, rr, cc] = 1.0
                x[0, 0, rr, cc] = level
            expected[rr, cc] = level
        h = oracle.hidden(x, z, lam, d, group_len=g)
        np.testing.assert_allclose(h[0, 0], expected, atol=1e-12)


# --------------------------------------------------------------------------
# Theorem 2: stability bound |h_i| <= sum_{j<=i} max|lambda_j x_j|
# --------------------------------------------------------------------------
def test_stability_bound():
    rng = np.random.default_rng(15)
    H, W = 17, 13
    x, z, lam, _ = rand_inputs(2, 2, H, W, rng, logit_std=3.0)
    for d in range(4):
        h = oracle.hidden(x, z[d], lam[d], d)
        drive = np.abs(lam[d] * x)
        for b in range(2):
            for c in range(2):
                acc = 0.0
                for rr, cc in scan_lines(d, H, W):
                    acc += drive[b, c, rr, cc].max()
                    assert np.abs(h[b, c, rr, cc]).max() <= acc + 1e-12


# --------------------------------------------------------------------------
# Linearity (H = G X; y linear in u and in lambda for fixed w)
# --------------------------------------------------------------------------
def test_linearity():
    rng = np.random.default_rng(16)
    x1, z, lam, u = rand_inputs(1, 2, 8, 6, rng)
    x2 = rng.normal(size=x1.shape)
    a, b = 1.7, -0.3
    for g in (0, 3):
        f = lambda xx, ll=lam, uu=u: oracle.forward(xx, z, ll, uu, g)
        np.testing.assert_allclose(f(a * x1 + b * x2), a * f(x1) + b * f(x2), atol=1e-11)
        u2 = [rng.normal(size=x1.shape) for _ in range(4)]
        mix = [a * p + b * q for p, q in zip(u, u2)]
        np.testing.assert_allclose(f(x1, uu=mix), a * f(x1) + b * f(x1, uu=u2), atol=1e-11)
        l2 = [rng.uniform(size=x1.shape) for _ in range(4)]
        mixl = [a * p + b * q for p, q in zip(lam, l2)]
        np.testing.assert_allclose(f(x1, ll=mixl), a * f(x1) + b * f(x1, ll=l2), atol=1e-11)


# --------------------------------------------------------------------------
# Special cases that reduce to textbook routines
# --------------------------------------------------------------------------
def test_single_column_is_prefix_sum():
    rng = np.random.default_rng(17)
    H = 23
    x = rng.normal(size=(1, 1, H, 1))
    z = rng.normal(size=(1, 1, 3, H, 1))
    lam = rng.uniform(size=(1, 1, H, 1))
    drive = (lam * x)[0, 0, :, 0]
    np.testing.assert_allclose(oracle.hidden(x, z, lam, 0)[0, 0, :, 0], np.cumsum(drive), atol=1e-12)
    np.testing.assert_allclose(oracle.hidden(x, z, lam, 1)[0, 0, :, 0],
                               np.cumsum(drive[::-1])[::-1], atol=1e-12)
    # the same plane scanned horizontally: every line is a single pixel
    np.testing.assert_allclose(oracle.hidden(x, z, lam, 2)[0, 0, :, 0], drive, atol=1e-15)


def test_single_row_is_prefix_sum_horizontally():
    rng = np.random.default_rng(18)
    W = 19
    x = rng.normal(size=(1, 1, 1, W))
    z = rng.normal(size=(1, 1, 3, 1, W))
    lam = rng.uniform(size=(1, 1, 1, W))
    drive = (lam * x)[0, 0, 0]
    np.testing.assert_allclose(oracle.hidden(x, z, lam, 2)[0, 0, 0], np.cumsum(drive), atol=1e-12)
    np.testing.assert_allclose(oracle.hidden(x, z, lam, 3)[0, 0, 0],
                               np.cumsum(drive[::-1])[::-1], atol=1e-12)


def test_group_len_one_is_pointwise():
    rng = np.random.default_rng(19)
    x, z, lam, u = rand_inputs(2, 2, 6, 7, rng)
    y = oracle.forward(x, z, lam, u, group_len=1)
    np.testing.assert_allclose(y, sum(u[d] * lam[d] * x for d in range(4)), atol=1e-13)


def test_group_len_at_least_L_is_global():
    rng = np.random.default_rng(20)
    x, z, lam, u = rand_inputs(1, 2, 9, 6, rng)
    y0 = oracle.forward(x, z, lam, u, 0)
    for g in (9, 10, 10**9):
        np.testing.assert_array_equal(oracle.forward(x, z, lam, u, g), y0)


def _tridiag_T(K):
    T = np.zeros((K, K))
    for k in range(K):
        nbrs = [kn for kn in (k - 1, k, k + 1) if 0 <= kn < K]
        for kn in nbrs:
            T[k, kn] = 1.0 / len(nbrs)
    return T


def test_equal_logits_give_matrix_powers():
    rng = np.random.default_rng(21)
    H, W = 8, 5
    x = rng.normal(size=(1, 1, H, W))
    lam = rng.uniform(size=(1, 1, H, W))
    z = np.full((1, 1, 3, H, W), 0.37)
    for d in range(4):
        K = W if d < 2 else H
        T = _tridiag_T(K)
        lines = scan_lines(d, H, W)
        drives = [(lam * x)[0, 0, rr, cc] for rr, cc in lines]
        h = oracle.hidden(x, z, lam, d)[0, 0]
        for i, (rr, cc) in enumerate(lines):
            ref = sum(np.linalg.matrix_power(T, i - j) @ drives[j] for j in range(i + 1))
            np.testing.assert_allclose(h[rr, cc], ref, atol=1e-12)


def test_dominant_slot_selects_the_named_neighbour():
    """Slot s with a huge logit (others tiny) copies the neighbour at offset s-1."""
    rng = np.random.default_rng(22)
    H, W = 6, 7
    x = rng.normal(size=(1, 1, H, W))
    lam = rng.uniform(size=(1, 1, H, W))
    for s in range(3):
        z = np.full((1, 1, 3, H, W), -40.0)
        z[:, :, s] = 40.0
        for d in range(4):
            h = oracle.hidden(x, z, lam, d)[0, 0]
            lines = scan_lines(d, H, W)
            K = W if d < 2 else H
            for i in range(1, len(lines)):
                rr, cc = lines[i]
                pr, pc = lines[i - 1]
                for k in range(1, K - 1):
                    ref = h[pr[k + s - 1], pc[k + s - 1]] + lam[0, 0, rr[k], cc[k]] * x[0, 0, rr[k], cc[k]]
                    assert abs(h[rr[k], cc[k]] - ref) < 1e-12


# --------------------------------------------------------------------------
# Direction conventions tied together by flips and transposition
# --------------------------------------------------------------------------
@pytest.mark.parametrize("g", [0, 3])
def test_direction_symmetries(g):
    rng = np.random.default_rng(23)
    H, W = 9, 6  # both divisible by 3 so local groups map onto each other
    x, z, lam, _ = rand_inputs(1, 2, H, W, rng)
    zz, ll = z[0], lam[0]
    h0 = oracle.hidden(x, zz, ll, 0, g)
    # d=1 on tensors flipped along H == d=0 flipped back
    h1 = oracle.hidden(x[:, :, ::-1], zz[:, :, :, ::-1], ll[:, :, ::-1], 1, g)
    np.testing.assert_allclose(h1[:, :, ::-1], h0, atol=1e-12)
    # d=2 on H<->W transposed tensors == d=0 transposed
    xt = np.swapaxes(x, 2, 3)
    zt = np.swapaxes(zz, 3, 4)
    lt = np.swapaxes(ll, 2, 3)
    h2 = oracle.hidden(xt, zt, lt, 2, g)
    np.testing.assert_allclose(np.swapaxes(h2, 2, 3), h0, atol=1e-12)
    # d=3 on tensors flipped along W == d=2 flipped back
    h2b = oracle.hidden(x, zz, ll, 2, g)
    h3 = oracle.hidden(x[:, :, :, ::-1], zz[:, :, :, :, ::-1], ll[:, :, :, ::-1], 3, g)
    np.testing.assert_allclose(h3[:, :, :, ::-1], h2b, atol=1e-12)


def test_local_groups_are_independent():
    rng = np.random.default_rng(24)
    H, W, g = 11, 10, 4
    x, z, lam, _ = rand_inputs(1, 1, H, W, rng)
    for d in range(4):
        h = oracle.hidden(x, z[d], lam[d], d, g)
        lines = scan_lines(d, H, W)
        gid = [dense_g.group_id(d, H, W, i, g) for i in range(len(lines))]
        target = gid[len(lines) // 2]
        x2, z2, l2 = x.copy(), z[d].copy(), lam[d].copy()
        for i, (rr, cc) in enumerate(lines):
            if gid[i] != target:
                x2[0, 0, rr, cc] += rng.normal(size=rr.size)
                z2[0, 0, :, rr, cc] += rng.normal(size=(rr.size, 3))
                l2[0, 0, rr, cc] = rng.uniform(size=rr.size)
        h2 = oracle.hidden(x2, z2, l2, d, g)
        for i, (rr, cc) in enumerate(lines):
            if gid[i] == target:
                np.testing.assert_array_equal(h2[0, 0, rr, cc], h[0, 0, rr, cc])


def test_rejects_bad_arguments():
    x = np.zeros((1, 1, 2, 2))
    z = np.zeros((1, 1, 3, 2, 2))
    with pytest.raises(ValueError):
        oracle.hidden(x, z, x, d=4)
    with pytest.raises(ValueError):
        oracle.hidden(x, z, x, d=0, group_len=-1)
