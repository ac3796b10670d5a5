"""GPU radix sort against the oracle's stable sort: the permutation (stable by
value, then original index) must match bit for bit, and so must the sorted values."""
import numpy as np
import pytest

import oracle
from structured_trainable_laplace_b200 import inputs
from tests.gpu_util import dev, host, laplex_or_fail

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return laplex_or_fail()


def check_sort(L, a):
    s, p = L.sort_anchors(dev(a))
    L.check()
    s_ref, p_ref = oracle.sort(a)
    np.testing.assert_array_equal(host(p), p_ref)
    assert np.array_equal(host(s).view(np.uint32), s_ref.view(np.uint32))


def test_small_with_ties():
    L = laplex_or_fail()
    check_sort(L, inputs.sym_small_ties(0)["a"])


@pytest.mark.parametrize("n", [1, 2, 3, 31, 4095, 4096, 4097, 12289, 100_003])
def test_ragged_sizes(L, n):
    a = np.random.default_rng(n).uniform(-50, 50, n).astype(np.float32)
    check_sort(L, a)


def test_heavy_ties_signed_zero_and_extremes(L):
    rng = np.random.default_rng(7)
    a = rng.integers(-5, 5, 50_001).astype(np.float32)
    a[rng.choice(a.size, 1000, replace=False)] = -0.0
    a[:6] = [np.finfo(np.float32).max, -np.finfo(np.float32).max, 1e-45, -1e-45, 1e-38, -0.0]
    check_sort(L, a)


def test_all_equal(L):
    check_sort(L, np.full(9000, 3.25, np.float32))


# up to 8192 anchors one CTA sorts the (key, index) composites in shared memory
@pytest.mark.parametrize("n", [5, 1000, 4096, 8191, 8192, 8193])
def test_single_cta_range_and_its_boundary(L, n):
    rng = np.random.default_rng(100 + n)
    a = rng.integers(-20, 20, n).astype(np.float32) * 0.5
    a[rng.random(n) < 0.1] = -0.0
    a[rng.random(n) < 0.05] = 0.0
    check_sort(L, a)
    check_sort(L, np.full(n, -7.5, np.float32))
    check_sort(L, np.linspace(1, -1, n).astype(np.float32))


def test_full_size_sort_of_the_2p24_workload(L):
    check_sort(L, inputs.sym_2p24_b16(0)["a"])


def test_bit_exact_past_2p24():
    """2^25 + 4097 anchors of the 10^9 workload's recipe (a ~ U[0, 0.05 n], fp32
    ulp 2 at the top: runs of ties), bit for bit against the oracle's stable sort:
    past 2^24 the radix passes run 8739 tiles and the lookback reaches further."""
    L = laplex_or_fail()
    check_sort(L, inputs.sym_extreme(4, n=(1 << 25) + 4097)["a"])


def test_nonfinite_anchor_sets_the_status_word(L):
    a = np.linspace(0, 1, 5000).astype(np.float32)
    a[1234] = np.nan
    L.sort_anchors(dev(a))
    with pytest.raises(L.LaplexError) as ei:
        L.check()
    assert ei.value.code == 4
    L.check()  # the word was reset
