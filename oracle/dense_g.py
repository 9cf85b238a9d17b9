"""Brute-force unrolled form of GSPN propagation -- TEST INFRASTRUCTURE ONLY.

The CSDN walkthrough "GSPN——在convolution基础上并行序列建模", section "方法",
writes the stacked hidden state as H = G X with a lower-triangular block matrix

    G_ij = (w_i w_{i-1} ... w_{j+1}) diag(lambda_j)   for j < i,
    G_ii = diag(lambda_i),

where w_r is the K x K tridiagonal matrix of scan line r.  This module builds
that matrix explicitly with numpy (no recurrence) for tiny planes and
multiplies it out.  It shares no code with ``gspn_oracle.cpp``; the tests use
it to pin the C++ loop's product order and lambda placement.

Local groups (section "全局与局部GSPN"): blocks G_ij whose lines i and j lie in
different groups are zero.  Line/pixel conventions are those stated in
``gspn_oracle.cpp``: direction 0 top->bottom, 1 bottom->top, 2 left->right,
3 right->left; logit slot s links to orthogonal offset s-1.
"""
from __future__ import annotations

import numpy as np


def _line_pixels(d: int, H: int, W: int, i: int):
    """(rows, cols) of scan line i of direction d, ordered by orthogonal index."""
    if d == 0:
        return np.full(W, i), np.arange(W)
    if d == 1:
        return np.full(W, H - 1 - i), np.arange(W)
    if d == 2:
        return np.arange(H), np.full(H, i)
    return np.arange(H), np.full(H, W - 1 - i)


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def line_matrix(z3: np.ndarray, d: int, i: int) -> np.ndarray:
    """K x K row-stochastic tridiagonal w_i of line i; z3 is one plane [3,H,W]."""
    _, H, W = z3.shape
    rows, cols = _line_pixels(d, H, W, i)
    K = rows.size
    w = np.zeros((K, K))
    for k in range(K):
        entries = {}
        for s in range(3):
            kn = k + s - 1
            if 0 <= kn < K:
                entries[kn] = _sigmoid(z3[s, rows[k], cols[k]])
        total = sum(entries.values())
        for kn, v in entries.items():
            w[k, kn] = v / total
    return w


def group_id(d: int, H: int, W: int, i: int, group_len: int) -> int:
    """Index of the propagation group holding scan line i (0 for global)."""
    L = H if d < 2 else W
    coord = i if d in (0, 2) else L - 1 - i
    return 0 if group_len <= 0 else coord // group_len


def dense_G(z3: np.ndarray, lam: np.ndarray, d: int, group_len: int = 0) -> np.ndarray:
    """The (L*K) x (L*K) matrix G of one plane; z3 [3,H,W], lam [H,W]."""
    _, H, W = z3.shape
    L = H if d < 2 else W
    K = W if d < 2 else H
    ws = [line_matrix(z3, d, i) for i in range(L)]
    lams = []
    for i in range(L):
        r, c = _line_pixels(d, H, W, i)
        lams.append(np.diag(lam[r, c]))
    G = np.zeros((L * K, L * K))
    for i in range(L):
        for j in range(i + 1):
            if group_id(d, H, W, i, group_len) != group_id(d, H, W, j, group_len):
                continue
            prod = np.eye(K)
            for r in range(j + 1, i + 1):  # w_i w_{i-1} ... w_{j+1}
                prod = ws[r] @ prod
            G[i * K:(i + 1) * K, j * K:(j + 1) * K] = prod @ lams[j]
    return G


def dense_hidden_plane(x: np.ndarray, z3: np.ndarray, lam: np.ndarray, d: int,
                       group_len: int = 0) -> np.ndarray:
    """h_d of one plane [H,W] as G @ vec(x), returned in image layout."""
    H, W = x.shape
    L = H if d < 2 else W
    xs = np.concatenate([x[_line_pixels(d, H, W, i)] for i in range(L)])
    hs = dense_G(z3, lam, d, group_len) @ xs
    K = W if d < 2 else H
    h = np.empty((H, W))
    for i in range(L):
        h[_line_pixels(d, H, W, i)] = hs[i * K:(i + 1) * K]
    return h


def dense_forward(x, wlogit, lam, u, group_len: int = 0) -> np.ndarray:
    """y = sum_d u_d * (G_d vec(x)) for float64 arrays x [B,C,H,W]."""
    x = np.asarray(x, dtype=np.float64)
    B, C, H, W = x.shape
    y = np.zeros_like(x)
    for d in range(4):
        z = np.asarray(wlogit[d], dtype=np.float64)
        la = np.asarray(lam[d], dtype=np.float64)
        ud = np.asarray(u[d], dtype=np.float64)
        for b in range(B):
            for c in range(C):
                y[b, c] += ud[b, c] * dense_hidden_plane(x[b, c], z[b, c], la[b, c], d, group_len)
    return y
