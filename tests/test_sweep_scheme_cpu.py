"""The halo schedule of the line-sweep kernel, modelled in numpy and checked
against the oracle (CPU only).

The line-sweep kernel (csrc/gspn_sweep.cu) never keeps one shared copy of a
scan line.  A chain's line is split over So CTAs, each CTA's window over warp
segments, and every segment recomputes its neighbours' edge positions:

* a segment holds 32 * kP consecutive window positions (kP = 2 per lane) and
  segments start every 32 * kP - 2 * kP positions, so neighbouring segments
  share one lane (kP positions) on each side;
* every kP steps each segment's outer lane is overwritten with the copy held
  by the neighbouring segment, where that position is interior;
* CTA sr owns positions [sr * Kc, (sr + 1) * Kc) (Kc a multiple of 8, at least
  16 when So > 1); its window starts 8 positions before the line's first
  position, or 16 before its owned range towards a neighbouring CTA, and
  every 16 steps the 16 positions on either side of the owned range are
  overwritten with the neighbouring CTA's copies.

The claim the kernel rests on: with this schedule every owned position is
exact at every step, whatever the values read beyond a segment's or a
window's end.  This model runs the schedule in fp64 with large random values
injected at every segment end, and compares the owned positions at every step
with the oracle's hidden state.  It checks the schedule and the window
geometry, not the CUDA code (the GPU parity tests do that).
"""
import numpy as np
import pytest

import oracle

KP = 2                      # positions per lane
SEG = 32 * KP               # positions per warp segment
STRIDE = SEG - 2 * KP       # segment spacing
EPOCH = KP                  # steps between warp refreshes
XHALO = 16                  # CTA halo width == steps between CTA refreshes
EDGE = 8                    # window margin at the ends of the line


def round_up(a, b):
    return (a + b - 1) // b * b


def model_hidden(x, w, lam, K, L, So, g, fwd, rng):
    """h of one vertical chain (lines = rows, positions = columns) under the
    line-sweep schedule; returns [L, K] with NaN where nothing was owned."""
    Kc = round_up(-(-K // So), 8)
    assert So == 1 or Kc >= XHALO
    margins = [(XHALO if sr > 0 else EDGE, XHALO if sr < So - 1 else EDGE) for sr in range(So)]
    span = max(ml + Kc + mr for ml, mr in margins)
    nw = -(-(span - 2 * KP) // STRIDE)
    win = STRIDE * nw + 2 * KP

    def inputs_at(i, a):
        """weights (3, n) and lambda*x (n) of line i at absolute positions a;
        positions outside the line carry zero inputs (finite weights)."""
        inside = (a >= 0) & (a < K)
        ac = np.clip(a, 0, K - 1)
        ww = np.where(inside, w[:, i, ac], 1.0 / 3.0)
        lx = np.where(inside, lam[i, ac] * x[i, ac], 0.0)
        return ww, lx

    ws = [sr * Kc - margins[sr][0] for sr in range(So)]
    # seg[sr][k]: copies of window positions [k*STRIDE, k*STRIDE + SEG)
    seg = [[np.zeros(SEG) for _ in range(nw)] for _ in range(So)]
    out = np.full((L, K), np.nan)
    rows = range(L) if fwd else range(L - 1, -1, -1)
    prev_row = None
    for s, i in enumerate(rows):
        start = s == 0 or (g > 0 and i // g != prev_row // g)
        prev_row = i
        for sr in range(So):
            for k in range(nw):
                a = ws[sr] + k * STRIDE + np.arange(SEG)
                ww, lx = inputs_at(i, a)
                old = seg[sr][k]
                garbage = rng.uniform(-1e6, 1e6, size=2)
                left = np.concatenate([[garbage[0]], old[:-1]])
                right = np.concatenate([old[1:], [garbage[1]]])
                new = lx if start else ww[0] * left + ww[1] * old + ww[2] * right + lx
                seg[sr][k] = new
                own0, own1 = sr * Kc, min(K, sr * Kc + Kc)
                rel = np.arange(SEG)
                core = (rel >= KP) & (rel < SEG - KP)
                sel = core & (a >= own0) & (a < own1)
                out[i, a[sel]] = new[sel]
        if (s + 1) % EPOCH != 0 or s + 1 >= L:
            continue
        # CTA refresh: 16 positions on each side of the owned range, from the
        # neighbouring CTA's interior copies (all read before any write)
        if So > 1 and (s + 1) % XHALO == 0:
            def copy_of(sr, pos):
                for k in range(nw):
                    r = pos - ws[sr] - k * STRIDE
                    if KP <= r < SEG - KP:
                        return seg[sr][k][r]
                raise AssertionError("position not interior in the sending CTA")
            updates = []
            for sr in range(So):
                own0 = sr * Kc
                halo = []
                if sr > 0:
                    halo += [(p, sr - 1) for p in range(own0 - XHALO, own0)]
                if sr < So - 1:
                    halo += [(p, sr + 1) for p in range(own0 + Kc, own0 + Kc + XHALO)]
                for p, src in halo:
                    updates.append((sr, p, copy_of(src, p)))
            for sr, p, v in updates:
                for k in range(nw):
                    r = p - ws[sr] - k * STRIDE
                    if 0 <= r < SEG:
                        seg[sr][k][r] = v
        # warp refresh: outer lanes from the neighbouring segments
        for sr in range(So):
            snap = [c.copy() for c in seg[sr]]
            for k in range(nw):
                if k > 0:
                    seg[sr][k][:KP] = snap[k - 1][STRIDE:STRIDE + KP]
                if k < nw - 1:
                    seg[sr][k][SEG - KP:] = snap[k + 1][SEG - KP - STRIDE:SEG - STRIDE]
    assert win >= span
    return out


CASES = [
    # (K, L, So, g)
    (96, 40, 1, 0),
    (130, 37, 1, 0),
    (300, 50, 2, 0),
    (301, 45, 2, 0),
    (520, 60, 4, 0),
    (777, 70, 4, 0),
    (129, 64, 8, 0),
    (1040, 40, 2, 0),
    (400, 66, 2, 7),
    (250, 50, 4, 16),
]


@pytest.mark.parametrize("K,L,So,g", CASES)
@pytest.mark.parametrize("d", [0, 1])
def test_sweep_schedule_is_exact(K, L, So, g, d):
    rng = np.random.default_rng(K * 31 + L + So + g + d)
    H, W = L, K
    x = rng.normal(size=(1, 1, H, W))
    z = rng.normal(size=(1, 1, 3, H, W))
    lam = rng.uniform(0.2, 1.0, size=(1, 1, H, W))
    ref = oracle.hidden(x, z, lam, d, g)[0, 0]
    w = oracle.weights(z, d)[0, 0]
    got = model_hidden(x[0, 0], w, lam[0, 0], K, L, So, g, d == 0, rng)
    assert not np.isnan(got).any(), "some position was owned by no CTA"
    assert np.abs(got - ref).max() <= 1e-9 * max(1.0, np.abs(ref).max())


def test_model_detects_a_broken_schedule():
    """Control: refreshing the warps every 2 * kP steps lets the injected
    garbage reach owned positions, so the check above is not vacuous."""
    global EPOCH
    keep = EPOCH
    EPOCH = 2 * KP
    try:
        rng = np.random.default_rng(3)
        K, L = 300, 30
        x = rng.normal(size=(1, 1, L, K))
        z = rng.normal(size=(1, 1, 3, L, K))
        lam = rng.uniform(0.2, 1.0, size=(1, 1, L, K))
        ref = oracle.hidden(x, z, lam, 0, 0)[0, 0]
        w = oracle.weights(z, 0)[0, 0]
        got = model_hidden(x[0, 0], w, lam[0, 0], K, L, 1, 0, True, rng)
        assert np.abs(got - ref).max() > 1.0
    finally:
        EPOCH = keep
