"""The decomposition behind the warm-start re-sort, checked in NumPy on the CPU
(no kernel involved): in any sequence of distinct composites c = (key, index), an
element above every composite before it and below every one after it sits at its
final rank, so sorting the others and writing them into the positions they hold
yields the sorted order.  The expected order is the oracle's stable sort."""
import numpy as np
import pytest

import oracle


def repair(a, perm_prev):
    """The warm path in plain NumPy: kept / displaced split, then placement."""
    n = a.size
    key = a[perm_prev].astype(np.float64)
    key[key == 0] = 0.0  # -0 == +0
    comp = list(zip(key.tolist(), perm_prev.tolist()))
    kept = np.zeros(n, bool)
    best = None
    suffix = [None] * (n + 1)
    for r in range(n - 1, -1, -1):
        suffix[r] = comp[r] if suffix[r + 1] is None else min(comp[r], suffix[r + 1])
    for r in range(n):
        above = best is None or comp[r] > best
        below = suffix[r + 1] is None or comp[r] < suffix[r + 1]
        kept[r] = above and below
        best = comp[r] if best is None else max(best, comp[r])
    out = perm_prev.copy()
    disp_pos = np.flatnonzero(~kept)
    disp = sorted(comp[r] for r in disp_pos)
    out[disp_pos] = [c[1] for c in disp]
    return out, kept


@pytest.mark.parametrize("seed", range(6))
def test_repair_gives_the_stable_order(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 400))
    a = rng.integers(0, max(2, n // 3), n).astype(np.float32) * 0.5   # many ties
    _, p_old = oracle.sort(a)
    b = (a + rng.normal(0, 0.6, n)).astype(np.float32)
    b[rng.random(n) < 0.05] = -0.0
    out, kept = repair(b, p_old)
    _, p_ref = oracle.sort(b)
    np.testing.assert_array_equal(out, p_ref)
    # kept elements are exactly where the stable order puts them
    np.testing.assert_array_equal(p_old[kept], p_ref[kept])


def test_one_far_move_displaces_only_what_it_passes():
    a = np.arange(50, dtype=np.float32)
    _, p_old = oracle.sort(a)
    b = a.copy()
    b[10] = 30.5
    out, kept = repair(b, p_old)
    np.testing.assert_array_equal(out, oracle.sort(b)[1])
    assert (~kept).sum() == 21  # the mover and the 20 it jumped over
