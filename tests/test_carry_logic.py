"""The sum form of the scan carries, checked in NumPy on the CPU (no kernel
involved).

A scan direction walks sorted (oriented) anchors u with inputs t.  The state at a
row is P (everything up to and including u_r, weighted exp(u_src - u_r)) and L (the
part whose source lies strictly before u_r) -- "LAPLEX: The FFT of Learnable Laplace
Kernels", technical summary section 2.2, the exact scan algebra, with the strict
sums that give sign(0) = 0 in the gradients.  Tiles publish their totals (L, P),
anchored at their last row.  The state entering tile k, anchored at the row just
before it (u_b), is then a plain sum over the earlier tiles j with end anchors u_j:

    P_in = sum_j e_j P_j,   L_in = sum_j (e_j P_j if u_j < u_b else L_j),
    e_j = exp(u_j - u_b)   (1 when u_j == u_b: the tile ends in a tie with u_b).

This is the form the small-side apply kernel, the symmetric range carries and the
block-wide lookback evaluate.  It is pinned here against the definition (a sum over
the sources) and against the sequential composition of the totals, with ties inside
tiles and across tile boundaries, in both scan directions, and with weights that
underflow far away (where the walk over the nearest tiles stops at the first zero
weight)."""
import math

import numpy as np
import pytest


def tile_totals(u, t, R):
    """(L, P) of each tile of R rows from a zero incoming state, by the recurrence
    P_r = d P_(r-1) + t_r, L_r = (u_r > u_(r-1)) ? d P_(r-1) : L_(r-1), d = exp(u_(r-1) - u_r)."""
    out = []
    for lo in range(0, u.size, R):
        L = P = 0.0
        for r in range(lo, min(u.size, lo + R)):
            if r == lo:
                L, P = 0.0, t[r]
                continue
            d = math.exp(u[r - 1] - u[r])
            L = d * P if u[r] > u[r - 1] else L
            P = d * P + t[r]
        out.append((L, P, u[min(u.size, lo + R) - 1]))
    return out


def definition(u, t, r0):
    """State entering row r0 (anchored at u[r0-1]) from its sources."""
    ub = u[r0 - 1]
    P = sum(math.exp(u[i] - ub) * t[i] for i in range(r0))
    L = sum(math.exp(u[i] - ub) * t[i] for i in range(r0) if u[i] < ub)
    return L, P


def sequential(tot, k):
    """Tiles 0 .. k-1 composed in order: A then B gives P = e P_A + P_B and
    L = (u_B > u_A) ? e P_A + L_B : L_A + L_B, e = exp(u_A - u_B)."""
    L, P, ua = tot[0]
    for Lb, Pb, ub in tot[1:k]:
        e = math.exp(ua - ub)
        L = e * P + Lb if ub > ua else L + Lb
        P = e * P + Pb
        ua = ub
    return L, P


def direct(tot, k, ub, nearest_first_stop=False):
    """The sum form; with nearest_first_stop, tiles are taken from k-1 down and the
    walk ends at the first weight that is exactly zero."""
    L = P = 0.0
    for j in range(k - 1, -1, -1):
        Lj, Pj, uj = tot[j]
        e = math.exp(uj - ub) if ub > uj else 1.0
        if nearest_first_stop and e == 0.0:
            break
        P += e * Pj
        L += e * Pj if ub > uj else Lj
    return L, P


def draw(rng, n, grid):
    u = np.sort(rng.uniform(0.0, n * 0.3, n))
    if grid:  # a coarse grid: tie runs inside tiles and across tile boundaries
        u = np.round(u / grid) * grid
    return u, rng.standard_normal(n)


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("R", [1, 3, 8])
def test_sum_form_equals_definition_and_fold(seed, R):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(R + 1, 160))
    u, t = draw(rng, n, grid=[None, 0.7, 2.5][seed % 3])
    for orient in (1.0, -1.0):  # left-to-right, and right-to-left on -u reversed
        uo = u if orient > 0 else -u[::-1]
        to = t if orient > 0 else t[::-1]
        tot = tile_totals(uo, to, R)
        for k in range(1, len(tot)):
            r0 = k * R
            Ld, Pd = definition(uo, to, r0)
            Ls, Ps = sequential(tot, k)
            Lx, Px = direct(tot, k, uo[r0 - 1])
            scale = sum(math.exp(uo[i] - uo[r0 - 1]) * abs(to[i]) for i in range(r0)) + 1e-300
            for got in ((Ls, Ps), (Lx, Px)):
                assert abs(got[0] - Ld) <= 1e-12 * scale and abs(got[1] - Pd) <= 1e-12 * scale, (k, got, Ld, Pd)


def test_all_equal_anchors_every_tile_ties():
    """Every tile ends in a tie with the boundary: weights 1, L collects only the
    tiles' own strict parts, which are zero; P is the plain sum."""
    u = np.full(40, 3.25)
    t = np.random.default_rng(3).standard_normal(40)
    tot = tile_totals(u, t, 4)
    for k in range(1, 10):
        L, P = direct(tot, k, u[4 * k - 1])
        assert L == 0.0
        assert abs(P - t[:4 * k].sum()) <= 1e-12 * np.abs(t).sum()


def test_a_dropped_tie_rule_is_caught():
    """Planted mistake: treating a tie at the boundary as a break (adding e P to L)
    changes L whenever a tile ends on u_b, which the definition sees."""
    u = np.array([0.0, 1.0, 2.0, 2.0, 2.0, 2.0, 3.0, 4.0])
    t = np.array([1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0, 8.0])
    tot = tile_totals(u, t, 2)
    k, ub = 3, u[5]  # tiles 0..2 end at 1.0, 2.0, 2.0; the boundary anchor is 2.0
    Ld, _ = definition(u, t, 2 * k)
    L, _ = direct(tot, k, ub)
    assert abs(L - Ld) < 1e-12
    wrong = sum(math.exp(uj - ub) * Pj for _, Pj, uj in tot[:k])
    assert abs(wrong - Ld) > 1.0


@pytest.mark.parametrize("seed", range(4))
def test_walk_may_stop_at_the_first_zero_weight(seed):
    """Sorted anchors make the weights fall with the distance, so once one is zero in
    fp64 every farther one is: stopping there gives the full sum exactly."""
    rng = np.random.default_rng(100 + seed)
    n, R = 600, 5
    u = np.cumsum(rng.uniform(0.5, 12.0, n))  # gaps wide enough to underflow within a few tiles
    t = rng.standard_normal(n)
    tot = tile_totals(u, t, R)
    stopped = 0
    for k in range(1, len(tot)):
        ub = u[k * R - 1]
        ws = [math.exp(uj - ub) if ub > uj else 1.0 for _, _, uj in tot[:k]][::-1]
        assert all(ws[i] >= ws[i + 1] for i in range(len(ws) - 1))
        full = direct(tot, k, ub)
        part = direct(tot, k, ub, nearest_first_stop=True)
        assert part == full
        stopped += ws[-1] == 0.0
    assert stopped > 0  # the stop rule was exercised
