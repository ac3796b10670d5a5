"""Symmetric operator on the GPU against the fp64 oracle: y = K x, gx = K g and
ga, elementwise within 1e-5 * twin + 1e-30 (twin = the same sums over |values|)."""
import numpy as np
import pytest

import oracle
from structured_trainable_laplace_b200 import inputs
from tests.gpu_util import dev, host, laplex_or_fail
from tests.parity import assert_close
from tests.sort_check import check_stable_sort

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return laplex_or_fail()


def run(L, a, x, g, saved=True):
    n, B = x.shape
    s, p = L.sort_anchors(dev(a))
    sv = L.saved_buffer("sym", n, 1, B, "cuda") if saved else None
    y = L.apply_sym(s, p, dev(x), saved=sv)
    gr = L.backward("sym", s, p, dev(x), dev(g), saved=sv)
    L.check()
    return host(y), host(gr["gx"]), host(gr["ga"])


def compare(L, a, x, g, saved=True, tag=""):
    y, gx, ga = run(L, a, x, g, saved)
    assert_close(y, oracle.sym_apply(a, x), oracle.sym_apply(a, x, twin=True), f"y {tag}")
    gx_ref, ga_ref = oracle.sym_backward(a, x, g)
    gx_tw, ga_tw = oracle.sym_backward(a, x, g, twin=True)
    assert_close(gx, gx_ref, gx_tw, f"gx {tag}")
    assert_close(ga, ga_ref, ga_tw, f"ga {tag}")


def test_small_workload_with_ties(L):
    w = inputs.sym_small_ties(0)
    compare(L, w["a"], w["x"], w["g"], tag="n4096")


@pytest.mark.parametrize("n,B", [(1, 1), (2, 3), (5000, 1), (70001, 4), (20000, 16), (9000, 40), (3000, 7),
                                 (33, 32), (12345, 2)])
@pytest.mark.parametrize("saved", [True, False])
def test_sizes_tiles_and_channel_groups(L, n, B, saved):
    w = inputs.symmetric(n, B, seed=n + B, tie_frac=0.05)
    compare(L, w["a"], w["x"], w["g"], saved, tag=f"n{n} B{B}")


def test_all_equal_anchors(L):
    rng = np.random.default_rng(3)
    a = np.full(7000, -2.5, np.float32)
    x, g = rng.standard_normal((7000, 3)).astype(np.float32), rng.standard_normal((7000, 3)).astype(np.float32)
    compare(L, a, x, g, tag="all equal")


def test_quantised_anchors_long_tie_runs(L):
    rng = np.random.default_rng(4)
    a = (rng.integers(0, 40, 60000) * 0.125).astype(np.float32)  # ~1500 per value: runs span tiles
    x, g = rng.standard_normal((60000, 2)).astype(np.float32), rng.standard_normal((60000, 2)).astype(np.float32)
    compare(L, a, x, g, tag="long runs")


def test_wide_gaps_and_underflow(L):
    rng = np.random.default_rng(5)
    a = np.concatenate([rng.uniform(0, 1, 3000), rng.uniform(500, 501, 3000), [1e4, -1e4]]).astype(np.float32)
    x, g = rng.standard_normal((a.size, 1)).astype(np.float32), rng.standard_normal((a.size, 1)).astype(np.float32)
    compare(L, a, x, g, tag="gaps")


def test_single_channel_past_the_unpermute_threshold(L):
    """B = 1 with n > 2^24: the sweeps write sorted-order outputs and the bucketed
    unpermute places them (y, gx, ga), with ties."""
    w = inputs.symmetric((1 << 24) + 4097, 1, seed=31, tie_frac=0.01)
    compare(L, w["a"], w["x"], w["g"], tag="n 2^24+4097 B1")


def test_full_size_2p24_b16(L):
    w = inputs.sym_2p24_b16(0)
    compare(L, w["a"], w["x"], w["g"], tag="2^24 x 16")


def test_full_size_1e9_b1(L):
    """n = 10^9 (B = 1) in the bench's configuration.  The sort is checked
    completely: its answer is unique (stable by value, then index), and the host
    checks every property that fixes it.  y, gx and ga are checked at 10^6 seeded
    sample indices against the oracle's windowed direct sums (the dropped mass,
    exp(-100) * sum |x| < 1e-30, is below the absolute tolerance)."""
    import os

    import torch
    free, _ = torch.cuda.mem_get_info()
    if free < 60e9:
        pytest.skip("needs ~60 GB of free device memory")
    w = inputs.sym_extreme(0)
    a, x, g = w["a"], w["x"], w["g"]
    n = a.size
    ad = dev(a)
    s, p = L.sort_anchors(ad)
    sv = L.saved_buffer("sym", n, 1, 1, "cuda")
    xd, gd = dev(x), dev(g)
    yd = L.apply_sym(s, p, xd, saved=sv)
    gr = L.backward("sym", s, p, xd, gd, saved=sv)
    L.check()
    s_h, p_h = host(s), host(p)
    y, gx, ga = host(yd), host(gr["gx"]), host(gr["ga"])
    del ad, s, p, sv, xd, gd, yd, gr
    torch.cuda.empty_cache()
    check_stable_sort(a, s_h, p_h)
    del s_h, p_h
    idx = np.random.default_rng(11).choice(n, 1_000_000, replace=False)
    threads = max(1, min(32, os.cpu_count() or 1))
    ref = oracle.sym_sampled(a, x, idx, g=g, window=100.0, threads=threads)
    assert np.all(ref["dropped"] < 1e-30)
    assert_close(y[idx], ref["y"], ref["y_twin"], "y 1e9")
    assert_close(ga[idx], ref["ga"], ref["ga_twin"], "ga 1e9")
    refg = oracle.sym_sampled(a, g, idx, window=100.0, threads=threads)
    assert_close(gx[idx], refg["y"], refg["y_twin"], "gx 1e9")
