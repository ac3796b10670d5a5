"""The bucketed single-channel permutation (out[perm[r]] = v[r] through two
destination splits and a window placement), modelled in NumPy on the CPU: the
index arithmetic the kernels rely on, with no kernel involved.

With b = ceil(log2 n), s2 = max(b - 16, 0) and s1 = s2 + 8, bucket q of the first
split holds exactly the destinations [q 2^s1, (q + 1) 2^s1) (a permutation has one
row per destination), so its pairs fill exactly those positions; when 2^s1 is a
multiple of the split tile, every second-split tile lies inside one first-split
bucket; and after the second split, window q holds exactly the destinations
[q 2^s2, (q + 1) 2^s2), so placing each window in its own buffer completes the
permutation."""
import numpy as np
import pytest

TILE = 4096


def split(p, v, shift, tile):
    """One split pass: per tile, pairs grouped by bucket p >> shift (low 8 bits within
    the tile's common upper bits); a cursor per bucket starts at bucket << shift."""
    n = p.size
    nb = ((n - 1) >> shift) + 1
    cursor = (np.arange(nb, dtype=np.int64) << shift)
    po, vo = np.empty_like(p), np.empty_like(v)
    for t0 in range(0, n, tile):
        pt, vt = p[t0:t0 + tile], v[t0:t0 + tile]
        b = pt.astype(np.int64) >> shift
        assert np.all((b >> 8) == (b[0] >> 8)), "a tile spans two upper-bit groups"
        order = np.argsort(b, kind="stable")  # any order inside a bucket is valid
        for bucket in np.unique(b):
            sel = order[b[order] == bucket]
            dst = cursor[bucket] + np.arange(sel.size)
            po[dst], vo[dst] = pt[sel], vt[sel]
            cursor[bucket] += sel.size
    return po, vo


def place(p, v, shift):
    n = p.size
    out = np.full(n, np.nan, np.float32)
    w = 1 << shift
    for w0 in range(0, n, w):
        cnt = min(w, n - w0)
        d = p[w0:w0 + cnt].astype(np.int64) - w0
        assert np.all((d >= 0) & (d < cnt)), "a window holds a destination outside it"
        out[w0 + d] = v[w0:w0 + cnt]
    return out


@pytest.mark.parametrize("n", [(1 << 20) + 4097, 3 << 19, 1 << 21])
def test_two_splits_and_windows_permute(n):
    rng = np.random.default_rng(n)
    perm = rng.permutation(n).astype(np.uint32)
    v = rng.standard_normal(n).astype(np.float32)
    bits = int(np.ceil(np.log2(n)))
    s2 = max(bits - 16, 0)
    s1 = s2 + 8
    # scaled down from the library's 2^24 threshold: the same bit arithmetic with a
    # smaller split tile keeps 2^s1 a multiple of the tile
    tile = min(TILE, 1 << s1)
    assert (1 << s1) % tile == 0
    p1, v1 = split(perm, v, s1, tile)
    for q in range(((n - 1) >> s1) + 1):
        lo, hi = q << s1, min(n, (q + 1) << s1)
        assert np.all((p1[lo:hi] >> s1) == q)
    p2, v2 = split(p1, v1, s2, tile)
    out = place(p2, v2, s2)
    ref = np.empty(n, np.float32)
    ref[perm] = v
    np.testing.assert_array_equal(out, ref)


@pytest.mark.parametrize("n", [(1 << 20) + 4097, 3 << 19])
def test_inverse_permutation_turns_the_gather_into_a_placement(n):
    """The gather xs[r] = x[perm[r]] of the single-channel path past 2^24 rows: the
    placement with positions as values builds inv (inv[perm[r]] = r), and the
    placement out[inv[i]] = x[i], which reads x in order, equals the gather."""
    rng = np.random.default_rng(n + 1)
    perm = rng.permutation(n).astype(np.uint32)
    x = rng.standard_normal(n).astype(np.float32)
    bits = int(np.ceil(np.log2(n)))
    s2 = max(bits - 16, 0)
    s1 = s2 + 8
    tile = min(TILE, 1 << s1)

    def placed(dest, vals):
        p1, v1 = split(dest, vals, s1, tile)
        p2, v2 = split(p1, v1, s2, tile)
        return place(p2, v2, s2)

    iota = np.arange(n, dtype=np.uint32).view(np.float32)  # positions as uint32 bits
    inv = placed(perm, iota).view(np.uint32)
    np.testing.assert_array_equal(inv[perm], np.arange(n, dtype=np.uint32))
    np.testing.assert_array_equal(placed(inv, x), x[perm])
