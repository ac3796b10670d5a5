"""Warm-start re-sort on the GPU against the oracle's stable sort of the moved
anchors: the permutation and the sorted values must match bit for bit whatever
path the call takes (already sorted, repaired, full sort)."""
import numpy as np
import pytest

import oracle
from structured_trainable_laplace_b200 import inputs
from tests.gpu_util import dev, host, laplex_or_fail

pytestmark = pytest.mark.gpu

SORTED, REPAIRED, FULL = 0, 1, 2


@pytest.fixture(scope="module")
def L():
    return laplex_or_fail()


def check_resort(L, a_new, perm_prev, expect_path=None):
    import torch
    path = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    s, p = L.resort_anchors(dev(a_new), dev(perm_prev), path)
    L.check()
    s_ref, p_ref = oracle.sort(a_new)
    np.testing.assert_array_equal(host(p), p_ref)
    assert np.array_equal(host(s).view(np.uint32), s_ref.view(np.uint32))
    got = int(path.item())
    assert got in (SORTED, REPAIRED, FULL)
    if expect_path is not None:
        assert got == expect_path, (got, expect_path)
    return got


def old_perm(a):
    return oracle.sort(a)[1]


def test_unchanged_anchors_take_the_sorted_path(L):
    a = inputs.symmetric(100_003, 1, seed=3, with_g=False)["a"]
    check_resort(L, a, old_perm(a), SORTED)


@pytest.mark.parametrize("step", [1e-4, 1e-3, 5e-3])
def test_small_moves_are_repaired(L, step):
    # mean spacing 0.05: steps of a tenth of it or less displace a small share
    a = inputs.symmetric(1 << 20, 1, seed=5, with_g=False)["a"]
    path = check_resort(L, inputs.moved(a, step, seed=11), old_perm(a))
    assert path in (SORTED, REPAIRED)


@pytest.mark.parametrize("step", [0.02, 0.1, 0.5])
def test_larger_moves_are_exact_on_either_path(L, step):
    a = inputs.symmetric(300_007, 1, seed=5, with_g=False)["a"]
    check_resort(L, inputs.moved(a, step, seed=13), old_perm(a))


def test_moves_far_beyond_the_spacing_fall_back_to_the_full_sort(L):
    a = inputs.symmetric(200_000, 1, seed=6, with_g=False)["a"]
    check_resort(L, inputs.moved(a, 50.0, seed=12), old_perm(a), FULL)


def test_unrelated_previous_order_falls_back(L):
    a = np.random.default_rng(8).uniform(0, 10, 70_001).astype(np.float32)
    perm_prev = np.random.default_rng(9).permutation(a.size).astype(np.uint32)
    check_resort(L, a, perm_prev, FULL)


def test_reversed_previous_order(L):
    a = np.linspace(0, 1, 50_000).astype(np.float32)
    check_resort(L, a, np.arange(a.size, dtype=np.uint32)[::-1].copy(), FULL)


@pytest.mark.parametrize("n", [1, 2, 3, 31, 4095, 4096, 4097, 12289])
def test_ragged_sizes(L, n):
    a = np.random.default_rng(n).uniform(0, 0.05 * n, n).astype(np.float32)
    check_resort(L, inputs.moved(a, 0.01, seed=n), old_perm(a))


def test_one_anchor_moved_across_many(L):
    # one anchor jumps over ~10^4 others: everything it passes is displaced
    a = np.arange(60_000, dtype=np.float32)
    perm_prev = old_perm(a)
    b = a.copy()
    b[100] = 10_100.5
    check_resort(L, b, perm_prev, REPAIRED)


def test_new_ties_order_by_index(L):
    # moves that create exact ties between anchors that were apart: equal values
    # must come out by ascending original index, not by their old order
    rng = np.random.default_rng(21)
    a = rng.integers(0, 2000, 30_000).astype(np.float32) + rng.uniform(0.01, 0.99, 30_000).astype(np.float32)
    perm_prev = old_perm(a)
    b = np.floor(a).astype(np.float32)
    check_resort(L, b, perm_prev)


def test_heavy_ties_and_signed_zero(L):
    rng = np.random.default_rng(22)
    a = rng.integers(-5, 5, 40_001).astype(np.float32)
    perm_prev = old_perm(a)
    b = a.copy()
    b[rng.choice(b.size, 500, replace=False)] = -0.0
    b[rng.choice(b.size, 500, replace=False)] += 1
    check_resort(L, b, perm_prev)


def test_previous_order_that_is_not_a_permutation(L):
    a = np.random.default_rng(23).uniform(0, 100, 20_000).astype(np.float32)
    p = old_perm(a)
    dup = p.copy()
    dup[500] = dup[501]  # a duplicate index
    check_resort(L, a, dup, FULL)
    big = p.copy()
    big[7] = 4_000_000_000  # out of range: clamped, then caught
    check_resort(L, a, big, FULL)


def test_full_size_2p24_workload_after_a_step(L):
    a = inputs.sym_2p24_b16(0)["a"]
    path = check_resort(L, inputs.moved(a, 0.01, seed=2), old_perm(a))
    assert path in (SORTED, REPAIRED)


def test_nonfinite_anchor_sets_the_status_word(L):
    a = np.linspace(0, 1, 5000).astype(np.float32)
    perm_prev = old_perm(a)
    b = a.copy()
    b[1234] = np.inf
    L.resort_anchors(dev(b), dev(perm_prev))
    with pytest.raises(L.LaplexError) as ei:
        L.check()
    assert ei.value.code == 4
    L.check()


def test_small_workspace_is_rejected(L):
    import ctypes
    import torch
    n = 10_000
    a = dev(np.zeros(n, np.float32))
    p = dev(np.arange(n, dtype=np.uint32))
    out_a = torch.empty(n, dtype=torch.float32, device="cuda")
    out_p = torch.empty(n, dtype=torch.int32, device="cuda")
    need = L.resort_workspace_size(n)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    code = L.lib().laplex_resort_anchors(ctypes.c_void_p(a.data_ptr()), n, ctypes.c_void_p(p.data_ptr()),
                                         ctypes.c_void_p(out_a.data_ptr()), ctypes.c_void_p(out_p.data_ptr()),
                                         ctypes.c_void_p(ws.data_ptr()), ws.numel(), None, None, None)
    assert code == 3
