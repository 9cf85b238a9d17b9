"""The halo schedule of the fused kernel, modelled in numpy and checked
against the oracle (CPU only).

The fused kernel (csrc/gspn_fused.cu) splits a chain over a team of S CTAs:
CTA r owns positions [r * Kc, (r + 1) * Kc) of the line (Kc a multiple of 64)
and also computes 32 positions on each side of them (its window has Kc + 64
positions; with S = 1 the window is the whole line rounded up to 64).  Every
32 steps a CTA sends its first and last 32 owned positions to its
neighbours, which overwrite their halos with them.  Between two exchanges a
halo position drifts from the exact value only from the window's ends
inward, one position per step, so the owned positions stay exact.

This model runs that schedule in fp64 with large random values read beyond
each window's ends and compares every owned position at every step with the
oracle's hidden state.  It checks the schedule, not the CUDA code (the GPU
parity tests do that).
"""
import numpy as np
import pytest

import oracle

HALO = 32  # halo width == steps between exchanges


def round_up(a, b):
    return (a + b - 1) // b * b


def model_hidden(x, w, lam, K, L, S, g, fwd, rng, halo=HALO):
    if S == 1:
        Kc = round_up(K, 64)
        kb = [0]
        npos = Kc
    else:
        Kc = round_up(-(-K // S), 64)
        kb = [r * Kc - halo for r in range(S)]
        npos = Kc + 2 * halo
    win = [np.zeros(npos) for _ in range(S)]
    out = np.full((L, K), np.nan)
    rows = range(L) if fwd else range(L - 1, -1, -1)
    prev = None
    for s, i in enumerate(rows):
        start = s == 0 or (g > 0 and i // g != prev // g)
        prev = i
        for r in range(S):
            a = kb[r] + np.arange(npos)
            inside = (a >= 0) & (a < K)
            ac = np.clip(a, 0, K - 1)
            ww = np.where(inside, w[:, i, ac], 1.0 / 3.0)
            lx = np.where(inside, lam[i, ac] * x[i, ac], 0.0)
            old = win[r]
            garbage = rng.uniform(-1e6, 1e6, size=2)
            left = np.concatenate([[garbage[0]], old[:-1]])
            right = np.concatenate([old[1:], [garbage[1]]])
            new = lx if start else ww[0] * left + ww[1] * old + ww[2] * right + lx
            win[r] = new
            own = (a >= r * Kc) & (a < min(K, (r + 1) * Kc))
            out[i, a[own]] = new[own]
        if S > 1 and (s + 1) % halo == 0 and s + 1 < L:
            snap = [v.copy() for v in win]
            for r in range(S):
                if r > 0:       # left halo <- the left neighbour's last owned positions
                    win[r][:halo] = snap[r - 1][Kc:Kc + halo]
                if r < S - 1:   # right halo <- the right neighbour's first owned positions
                    win[r][Kc + halo:] = snap[r + 1][halo:2 * halo]
    return out


CASES = [
    # (K, L, S, g)
    (96, 70, 1, 0),
    (700, 80, 2, 0),
    (701, 75, 2, 0),
    (1500, 70, 4, 0),
    (2100, 66, 8, 0),
    (1201, 90, 4, 100),
    (300, 100, 2, 33),
    (64, 40, 4, 0),   # narrow: trailing CTAs own nothing
]


@pytest.mark.parametrize("K,L,S,g", CASES)
@pytest.mark.parametrize("d", [0, 1])
def test_fused_schedule_is_exact(K, L, S, g, d):
    rng = np.random.default_rng(K * 7 + L + S + g + d)
    x = rng.normal(size=(1, 1, L, K))
    z = rng.normal(size=(1, 1, 3, L, K))
    lam = rng.uniform(0.2, 1.0, size=(1, 1, L, K))
    ref = oracle.hidden(x, z, lam, d, g)[0, 0]
    w = oracle.weights(z, d)[0, 0]
    got = model_hidden(x[0, 0], w, lam[0, 0], K, L, S, g, d == 0, rng)
    assert not np.isnan(got).any(), "some position was owned by no CTA"
    assert np.abs(got - ref).max() <= 1e-9 * max(1.0, np.abs(ref).max())


def test_model_detects_a_broken_schedule():
    """Control: a 16-wide halo exchanged every 32 steps lets the values read
    beyond the windows reach owned positions."""
    rng = np.random.default_rng(5)
    K, L, S = 700, 80, 2
    x = rng.normal(size=(1, 1, L, K))
    z = rng.normal(size=(1, 1, 3, L, K))
    lam = rng.uniform(0.2, 1.0, size=(1, 1, L, K))
    ref = oracle.hidden(x, z, lam, 0, 0)[0, 0]
    w = oracle.weights(z, 0)[0, 0]

    def broken(*args):
        # windows with 16-wide halos, still exchanged every 32 steps
        Kc = round_up(-(-K // S), 64)
        out = np.full((L, K), np.nan)
        kb = [r * Kc - 16 for r in range(S)]
        npos = Kc + 32
        win = [np.zeros(npos) for _ in range(S)]
        for i in range(L):
            for r in range(S):
                a = kb[r] + np.arange(npos)
                inside = (a >= 0) & (a < K)
                ac = np.clip(a, 0, K - 1)
                ww = np.where(inside, w[:, i, ac], 1.0 / 3.0)
                lx = np.where(inside, lam[0, 0, i, ac] * x[0, 0, i, ac], 0.0)
                old = win[r]
                g2 = rng.uniform(-1e6, 1e6, size=2)
                left = np.concatenate([[g2[0]], old[:-1]])
                right = np.concatenate([old[1:], [g2[1]]])
                win[r] = lx if i == 0 else ww[0] * left + ww[1] * old + ww[2] * right + lx
                own = (a >= r * Kc) & (a < min(K, (r + 1) * Kc))
                out[i, a[own]] = win[r][own]
            if (i + 1) % 32 == 0 and i + 1 < L:
                snap = [v.copy() for v in win]
                win[1][:16] = snap[0][Kc:Kc + 16]
                win[0][Kc + 16:] = snap[1][16:32]
        return out

    got = broken()
    assert np.abs(got - ref).max() > 1.0
