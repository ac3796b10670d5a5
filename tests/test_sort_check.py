"""The host-side stable-sort checker (used on the 10^9-anchor permutation) against
the oracle's stable sort, and planted mistakes that it must catch."""
import numpy as np
import pytest

import oracle
from tests.sort_check import check_stable_sort


def _draw(n=50_000, seed=0):
    rng = np.random.default_rng(seed)
    a = (rng.integers(-200, 200, n) * 0.25).astype(np.float32)  # many ties
    a[rng.choice(n, 500, replace=False)] = -0.0
    return a


@pytest.mark.parametrize("chunk", [1 << 26, 4096, 1000])
def test_accepts_the_stable_sort(chunk):
    a = _draw()
    s, p = oracle.sort(a)
    check_stable_sort(a, s, p, chunk=chunk)


def _fails(a, s, p):
    with pytest.raises(AssertionError):
        check_stable_sort(a, s, p, chunk=997)


def test_catches_planted_mistakes():
    a = _draw()
    s, p = oracle.sort(a)
    # two tied anchors swapped (values still sorted): tie order broken
    r = int(np.flatnonzero(s[1:] == s[:-1])[0])
    q = p.copy()
    q[r], q[r + 1] = q[r + 1], q[r]
    _fails(a, s, q)
    # a tie swap across a chunk boundary
    r = int(np.flatnonzero((s[1:] == s[:-1]) & (np.arange(1, a.size) % 997 == 0))[0])
    q = p.copy()
    q[r], q[r + 1] = q[r + 1], q[r]
    _fails(a, s, q)
    # a duplicated index (not a permutation), values kept consistent
    q = p.copy()
    q[10] = q[11]
    _fails(a, s, q)
    # an entry out of range
    q = p.copy()
    q[5] = a.size
    _fails(a, s, q)
    # two distinct values swapped in both arrays (a[perm] still matches, order broken)
    r = int(np.flatnonzero(s[1:] > s[:-1])[0])
    q, t = p.copy(), s.copy()
    q[r], q[r + 1] = q[r + 1], q[r]
    t[r], t[r + 1] = t[r + 1], t[r]
    _fails(a, t, q)
    # a sorted value that does not match its anchor
    t = s.copy()
    t[123] = np.nextafter(t[123], np.float32(np.inf))
    _fails(a, t, p)
    # -0.0 and +0.0 are the same anchor value
    t = s.copy()
    t[t == 0] = -0.0
    check_stable_sort(a, t, p)
