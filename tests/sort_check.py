"""Complete host-side check of a stable anchor sort, for sizes the oracle's sort
cannot take in a test (n up to 10^9).

The sort the pages start from ("after sorting the anchors", technical summary
section 2.2) is taken stable by (value, original index), which makes its answer
unique: (a_sorted, perm) is that answer if and only if
  1. perm is a permutation of 0 .. n-1,
  2. a_sorted[r] == a[perm[r]] bit for bit (with -0.0 read as +0.0),
  3. a_sorted is nondecreasing, and
  4. perm ascends inside every run of equal values.
The arrays are walked in chunks so that the temporaries stay small."""
from __future__ import annotations

import numpy as np

_CHUNK = 1 << 26


def _canon_bits(v: np.ndarray) -> np.ndarray:
    """fp32 bit patterns with -0.0 replaced by +0.0."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).copy()
    b[b == 0x80000000] = 0
    return b


def check_stable_sort(a: np.ndarray, a_sorted: np.ndarray, perm: np.ndarray, chunk: int = _CHUNK) -> None:
    """Raise AssertionError unless (a_sorted, perm) is the stable sort of a."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    n = a.shape[0]
    assert a_sorted.shape == (n,) and perm.shape == (n,), "shapes"
    perm = np.ascontiguousarray(perm, dtype=np.uint32)
    seen = np.zeros(n, dtype=bool)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        p = perm[s:e]
        assert int(p.max(initial=0)) < n, f"perm entry >= n in [{s}, {e})"
        seen[p] = True
        got = _canon_bits(a_sorted[s:e])
        want = _canon_bits(a[p])
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, f"a_sorted[r] != a[perm[r]] at r = {s + int(bad[0])}"
        # pairs (r, r + 1) for r in [s, e), the last one reaching into the next chunk
        e1 = min(n, e + 1)
        v = a_sorted[s:e1].astype(np.float32)
        q = perm[s:e1]
        dec = np.flatnonzero(v[1:] < v[:-1])
        assert dec.size == 0, f"a_sorted decreases at r = {s + int(dec[0])}"
        tie = v[1:] == v[:-1]
        order = np.flatnonzero(tie & (q[1:] <= q[:-1]))
        assert order.size == 0, f"equal anchors out of index order at r = {s + int(order[0])}"
    missing = np.flatnonzero(~seen)
    assert missing.size == 0, f"perm misses index {int(missing[0])} (not a permutation)"
