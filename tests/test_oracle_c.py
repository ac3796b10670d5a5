"""Pins for the C fp64 oracle: against the dense definitions (themselves pinned in
test_oracle_dense.py) on small inputs with many ties, and at sizes where no
dense matrix fits against independent facts: the closed form on a uniform grid,
a Toeplitz product through NumPy's FFT, the tridiagonal inverse of the kernel of
distinct 1-D anchors, NumPy's stable argsort, and the gradient invariances."""
import math

import numpy as np
import pytest

import oracle
from oracle import dense
from structured_trainable_laplace_b200 import inputs
from tests.golden import fixtures
from tests.test_oracle_dense import grid_closed_form, toeplitz_fft_matvec


def rel(u, v):
    return float(np.max(np.abs(u - v)) / max(1e-300, np.max(np.abs(v))))


def tied(rng, n, step=0.5, m=12):
    return (rng.integers(0, m, n) * step).astype(np.float32)


def test_worked_examples():
    G = fixtures.load()
    s = G["sym"]
    np.testing.assert_allclose(oracle.sym_apply(s["a"], s["x"])[:, 0], s["y"], rtol=1e-14)
    gx, ga = oracle.sym_backward(s["a"], s["x"], s["g"])
    np.testing.assert_allclose(gx[:, 0], s["gx"], rtol=1e-14)
    np.testing.assert_allclose(ga, s["ga"], rtol=1e-13, atol=1e-15)
    p = G["phased"]
    np.testing.assert_allclose(oracle.rect_apply(p["a"], p["b"], p["x"], p["phi"], p["psi"])[:, 0], p["y"],
                               rtol=1e-14)
    gr = oracle.rect_backward(p["a"], p["b"], p["x"], p["g"], p["phi"], p["psi"])
    for key in ("ga", "gb", "gphi", "gpsi"):
        np.testing.assert_allclose(gr[key], p[key], rtol=1e-13, err_msg=key)
    q = G["gram"]
    np.testing.assert_allclose(oracle.gram_apply(q["a"], q["b"], q["D"], q["v"])[:, 0], q["y"], rtol=1e-14)
    np.testing.assert_allclose(oracle.gram_backward_D(q["a"], q["b"], q["v"], q["g"]), q["gD"], rtol=1e-14)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_symmetric_matches_dense(seed):
    rng = np.random.default_rng(seed)
    n, B = 61, 3
    a = tied(rng, n)
    x, g = rng.standard_normal((n, B)).astype(np.float32), rng.standard_normal((n, B)).astype(np.float32)
    for twin in (False, True):
        assert rel(oracle.sym_apply(a, x, twin), dense.sym_apply(a, x, twin)) < 1e-14
        gx, ga = oracle.sym_backward(a, x, g, twin)
        dgx, dga = dense.sym_backward(a, x, g, twin)
        assert rel(gx, dgx) < 1e-14 and rel(ga, dga) < 1e-13


@pytest.mark.parametrize("phased", [False, True])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("seed", [0, 1])
def test_rectangular_matches_dense(phased, transpose, seed):
    rng = np.random.default_rng(10 + seed)
    n, k, B = 47, 19, 2
    a, b = tied(rng, n), tied(rng, k)  # ties inside a, inside b and between them
    phi = rng.uniform(0, 2 * np.pi, n).astype(np.float32) if phased else None
    psi = rng.uniform(0, 2 * np.pi, k).astype(np.float32) if phased else None
    x = rng.standard_normal(((n if transpose else k), B)).astype(np.float32)
    g = rng.standard_normal(((k if transpose else n), B)).astype(np.float32)
    for twin in (False, True):
        assert rel(oracle.rect_apply(a, b, x, phi, psi, transpose, twin),
                   dense.rect_apply(a, b, x, phi, psi, transpose, twin)) < 1e-13
        o = oracle.rect_backward(a, b, x, g, phi, psi, transpose, twin)
        d = dense.rect_backward(a, b, x, g, phi, psi, transpose, twin)
        for key in d:
            assert rel(o[key], d[key]) < 1e-13, (key, twin)


def test_gram_matches_dense():
    rng = np.random.default_rng(20)
    a, b = tied(rng, 40, 0.25, 30), tied(rng, 9, 0.25, 30)
    D = rng.uniform(0.1, 2, 9).astype(np.float32)
    v, g = rng.standard_normal((40, 3)).astype(np.float32), rng.standard_normal((40, 3)).astype(np.float32)
    y, w = oracle.gram_apply(a, b, D, v, return_w=True)
    assert rel(y, dense.gram_apply(a, b, D, v)) < 1e-13
    assert rel(w, dense.rect_apply(a, b, v, transpose=True)) < 1e-13
    assert rel(oracle.gram_apply(a, b, D, v, twin=True), dense.gram_apply(a, b, D, v, twin=True)) < 1e-13
    assert rel(oracle.gram_backward_D(a, b, v, g), dense.gram_backward_D(a, b, v, g)) < 1e-13


def test_gram_full_backward_matches_dense():
    """The composed C evaluation of every Gram gradient against the dense
    definition, with ties inside a, inside b and between them.  The composition
    rounds A^T v and A^T g to fp32 between its passes (relative 6e-8)."""
    rng = np.random.default_rng(22)
    a, b = tied(rng, 50, 0.25, 30), tied(rng, 11, 0.25, 30)
    D = rng.uniform(0.1, 2, 11).astype(np.float32)
    v, g = rng.standard_normal((50, 2)).astype(np.float32), rng.standard_normal((50, 2)).astype(np.float32)
    got, ref = oracle.gram_backward(a, b, D, v, g), dense.gram_backward(a, b, D, v, g)
    tw = dense.gram_backward(a, b, D, v, g, twin=True)
    for key in ("gv", "ga", "gb", "gD"):
        assert np.all(np.abs(got[key] - ref[key]) <= 1e-6 * tw[key] + 1e-12), key
    got_tw = oracle.gram_backward(a, b, D, v, g, twin=True)
    for key in ("gv", "ga", "gb", "gD"):
        assert np.all(got_tw[key] >= np.abs(ref[key]) * (1 - 1e-6) - 1e-12), key


def test_sort_matches_numpy_stable_argsort():
    rng = np.random.default_rng(21)
    a = tied(rng, 5000, 0.125, 64)
    a[::7] = -0.0
    a[3::11] = 0.0
    s, p = oracle.sort(a)
    np.testing.assert_array_equal(p, np.argsort(a, kind="stable").astype(np.uint32))
    assert np.all(np.diff(s) >= 0)
    assert np.array_equal(np.sort(p), np.arange(5000, dtype=np.uint32))
    assert not np.any(np.signbit(s[s == 0]))  # -0 comes back as +0


def test_nonfinite_anchor_is_an_error():
    a = np.array([0.0, np.nan, 1.0], np.float32)
    with pytest.raises(ValueError, match="non-finite"):
        oracle.sym_apply(a, np.ones(3, np.float32))
    with pytest.raises(ValueError, match="non-finite"):
        oracle.sort(np.array([np.inf, 0.0], np.float32))


def test_closed_form_on_a_large_grid():
    n, delta = 1 << 18, 0.0625
    a = (np.arange(1, n + 1) * delta).astype(np.float32)
    y = oracle.sym_apply(np.random.default_rng(0).permutation(a), np.ones(n, np.float32))
    # the permutation moves rows along with anchors; compare in sorted order
    order = np.argsort(np.random.default_rng(0).permutation(a), kind="stable")
    np.testing.assert_allclose(y[order, 0], grid_closed_form(n, delta), rtol=1e-12)


def test_toeplitz_fft_on_a_large_grid():
    n, delta = 1 << 18, 0.125
    a = (np.arange(n) * delta).astype(np.float32)
    x = np.random.default_rng(22).standard_normal(n).astype(np.float32)
    ref = toeplitz_fft_matvec(np.exp(-np.arange(n) * delta), x.astype(np.float64))
    np.testing.assert_allclose(oracle.sym_apply(a, x)[:, 0], ref, rtol=1e-9, atol=1e-10)


def ou_precision_apply(s, y):
    """Q y for Q = K^-1 of sorted distinct anchors s (an AR(1)/Ornstein-Uhlenbeck chain):
    rho_i = exp(-(s_{i+1} - s_i)); Q is tridiagonal with
    Q_ii = 1/(1-rho_{i-1}^2) + rho_i^2/(1-rho_i^2) (missing terms are 0 at the ends... with
    rho_0 = rho_n = 0 this gives Q_11 = 1/(1-rho_1^2)), Q_{i,i+1} = -rho_i/(1-rho_i^2)."""
    rho = np.exp(-np.diff(s.astype(np.float64)))
    inv = 1.0 / (1.0 - rho ** 2)
    diag = np.ones_like(s, dtype=np.float64)
    diag[1:] += rho ** 2 * inv  # 1/(1-rho_{i-1}^2) = 1 + rho_{i-1}^2/(1-rho_{i-1}^2)
    diag[:-1] += rho ** 2 * inv
    off = -rho * inv
    out = diag[:, None] * y
    out[:-1] += off[:, None] * y[1:]
    out[1:] += off[:, None] * y[:-1]
    return out


def test_tridiagonal_inverse_formula_against_numpy_inverse():
    rng = np.random.default_rng(23)
    s = np.sort(rng.uniform(0, 10, 60))
    K = dense.kernel(s, s)
    np.testing.assert_allclose(ou_precision_apply(s, np.eye(60)), np.linalg.inv(K), atol=1e-8)


def test_tridiagonal_inverse_recovers_x_at_large_n():
    w = inputs.symmetric(1 << 18, 2, seed=3)
    keep = np.unique(w["a"], return_index=True)[1]  # drop fp32 ties: the formula needs distinct anchors
    a, x = w["a"][keep], w["x"][keep]
    s, p = oracle.sort(a)
    assert np.all(np.diff(s) > 0)
    y = oracle.sym_apply(a, x)
    back = ou_precision_apply(s, y[p.astype(np.int64)])
    np.testing.assert_allclose(back, x[p.astype(np.int64)], rtol=1e-9, atol=1e-9)


def test_windowed_sampling_matches_full_oracle():
    w = inputs.symmetric(1 << 16, 2, seed=4, tie_frac=0.05)
    a, x, g = w["a"], w["x"], w["g"]
    idx = np.random.default_rng(5).choice(a.shape[0], 300, replace=False)
    smp = oracle.sym_sampled(a, x, idx, g=g, window=100.0)
    y = oracle.sym_apply(a, x)
    _, ga = oracle.sym_backward(a, x, g)
    assert np.all(smp["dropped"] < 1e-30)
    twin = oracle.sym_apply(a, x, twin=True)[idx]
    assert np.all(np.abs(smp["y"] - y[idx]) <= 1e-12 * twin)
    _, ga_twin = oracle.sym_backward(a, x, g, twin=True)
    assert np.all(np.abs(smp["ga"] - ga[idx]) <= 1e-12 * ga_twin[idx])
    np.testing.assert_allclose(smp["ga_twin"], ga_twin[idx], rtol=1e-12)
    np.testing.assert_allclose(smp["y_twin"], twin, rtol=1e-12)


def test_gradient_invariances_at_scale_with_ties():
    w = inputs.sym_small_ties(0)
    _, ga = oracle.sym_backward(w["a"], w["x"], w["g"])
    assert abs(ga.sum()) < 1e-11 * np.abs(ga).sum()
    h = inputs.phased_head(4096, 64, 4, seed=1)
    gr = oracle.rect_backward(h["a"], h["b"], h["x"], h["h"], h["phi"], h["psi"], transpose=True)
    assert abs(gr["ga"].sum() + gr["gb"].sum()) < 1e-11 * np.abs(gr["ga"]).sum()
    assert abs(gr["gphi"].sum() + gr["gpsi"].sum()) < 1e-11 * np.abs(gr["gphi"]).sum()


def test_degenerate_sizes_and_all_equal_anchors():
    x = np.array([[2.5, -1.0]], np.float32)
    np.testing.assert_array_equal(oracle.sym_apply(np.array([3.0], np.float32), x), x.astype(np.float64))
    gx, ga = oracle.sym_backward(np.array([3.0], np.float32), x, x)
    assert ga[0] == 0.0
    rng = np.random.default_rng(24)
    xa, ga_ = rng.standard_normal((9, 2)).astype(np.float32), rng.standard_normal((9, 2)).astype(np.float32)
    a = np.full(9, 1.5, np.float32)
    np.testing.assert_allclose(oracle.sym_apply(a, xa), np.tile(xa.astype(np.float64).sum(0), (9, 1)), rtol=1e-14)
    gx, ga = oracle.sym_backward(a, xa, ga_)
    np.testing.assert_array_equal(ga, 0.0)
    # k = 1 rectangular: a single output anchor collects everything
    z = oracle.rect_apply(np.array([0.0, 1.0], np.float32), np.array([1.0], np.float32), xa[:2], transpose=True)
    np.testing.assert_allclose(z[0], math.exp(-1) * xa[0].astype(np.float64) + xa[1], rtol=1e-14)
