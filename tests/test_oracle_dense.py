"""Pins for the dense fp64 definitions (oracle.dense) against facts that do not
come from the definitions' own code: hand-derived worked examples, the closed form
of the recurrence on a uniform grid, a Toeplitz product through NumPy's FFT,
positive-definiteness of the Laplace kernel, central finite differences of the
forward, and the exact invariances of the gradients."""
import math

import numpy as np
import pytest

from oracle import dense
from tests.golden import fixtures

GOLD = fixtures.load()


def test_worked_example_symmetric():
    s = GOLD["sym"]
    np.testing.assert_allclose(dense.sym_apply(s["a"], s["x"])[:, 0], s["y"], rtol=1e-14)
    gx, ga = dense.sym_backward(s["a"], s["x"], s["g"])
    np.testing.assert_allclose(gx[:, 0], s["gx"], rtol=1e-14)
    np.testing.assert_allclose(ga, s["ga"], rtol=1e-13, atol=1e-15)


def test_worked_example_phased():
    s = GOLD["phased"]
    y = dense.rect_apply(s["a"], s["b"], s["x"], s["phi"], s["psi"])
    np.testing.assert_allclose(y[:, 0], s["y"], rtol=1e-14)
    gr = dense.rect_backward(s["a"], s["b"], s["x"], s["g"], s["phi"], s["psi"])
    for key in ("ga", "gb", "gphi", "gpsi"):
        np.testing.assert_allclose(gr[key], s[key], rtol=1e-13, err_msg=key)
    np.testing.assert_allclose(gr["gx"][:, 0], s["gx"], rtol=1e-13)


def test_worked_example_gram():
    s = GOLD["gram"]
    np.testing.assert_allclose(dense.gram_apply(s["a"], s["b"], s["D"], s["v"])[:, 0], s["y"], rtol=1e-14)
    np.testing.assert_allclose(dense.gram_backward_D(s["a"], s["b"], s["v"], s["g"]), s["gD"], rtol=1e-14)


def grid_closed_form(n, delta):
    """x = 1 on a_i = i*delta: y_i = (1-q^i)/(1-q) + (1-q^(n-i+1))/(1-q) - 1, q = e^-delta (1-based i)."""
    q = math.exp(-delta)
    i = np.arange(1, n + 1, dtype=np.float64)
    return (1 - q ** i) / (1 - q) + (1 - q ** (n - i + 1)) / (1 - q) - 1


@pytest.mark.parametrize("n,delta", [(1, 0.5), (7, 0.25), (300, 0.0625), (1000, 2.0)])
def test_closed_form_on_grid(n, delta):
    a = (np.arange(1, n + 1) * delta).astype(np.float32)
    np.testing.assert_allclose(dense.sym_apply(a, np.ones(n))[:, 0], grid_closed_form(n, delta), rtol=1e-13)


def toeplitz_fft_matvec(col, x):
    """Symmetric Toeplitz matrix (first column col) times x through a circulant embedding."""
    n = col.shape[0]
    c = np.concatenate([col, [0.0], col[:0:-1]])
    xp = np.concatenate([x, np.zeros(n)])
    return np.fft.irfft(np.fft.rfft(c) * np.fft.rfft(xp), 2 * n)[:n]


def test_grid_anchors_make_a_toeplitz_product():
    n, delta = 513, 0.125
    a = (np.arange(n) * delta).astype(np.float32)
    x = np.random.default_rng(3).standard_normal(n)
    col = np.exp(-np.arange(n) * delta)
    np.testing.assert_allclose(dense.sym_apply(a, x)[:, 0], toeplitz_fft_matvec(col, x), rtol=1e-9, atol=1e-12)


def test_distinct_anchors_give_positive_definite_kernel():
    rng = np.random.default_rng(4)
    a = np.unique(rng.uniform(0, 20, 200).astype(np.float32))
    K = dense.kernel(a, a)
    np.linalg.cholesky(K)
    for _ in range(5):
        x = rng.standard_normal(a.shape[0])
        assert x @ dense.sym_apply(a, x)[:, 0] > 0


def test_tied_anchors_make_a_singular_kernel():
    a = np.array([0.0, 1.0, 1.0, 2.5], np.float32)
    x = np.array([0.0, 1.0, -1.0, 0.0])
    np.testing.assert_allclose(dense.sym_apply(a, x)[:, 0], 0.0, atol=1e-15)


def test_adjoint_identity():
    rng = np.random.default_rng(5)
    a, b = rng.uniform(0, 5, 30), rng.uniform(0, 5, 11)
    phi, psi = rng.uniform(0, 6, 30), rng.uniform(0, 6, 11)
    x, g = rng.standard_normal((11, 3)), rng.standard_normal((30, 3))
    for ph in (False, True):
        P = (phi, psi) if ph else (None, None)
        lhs = np.sum(g * dense.rect_apply(a, b, x, *P))
        rhs = np.sum(dense.rect_apply(a, b, g, *P, transpose=True) * x)
        assert abs(lhs - rhs) <= 1e-12 * abs(lhs) + 1e-12


def test_zero_phases_reduce_to_unphased():
    rng = np.random.default_rng(6)
    a, b = rng.uniform(0, 5, 20), rng.uniform(0, 5, 9)
    x = rng.standard_normal((9, 2))
    z = np.zeros
    np.testing.assert_allclose(dense.rect_apply(a, b, x, z(20), z(9)), dense.rect_apply(a, b, x), rtol=1e-15)
    c = 1.25
    np.testing.assert_allclose(dense.rect_apply(a, b, x, z(20) + c, z(9) + c), dense.rect_apply(a, b, x),
                               rtol=1e-13)


def separated(rng, n, lo, hi, gap=1e-2):
    """Anchors whose nearest neighbours are more than `gap` apart (|t| smooth there)."""
    while True:
        a = np.sort(rng.uniform(lo, hi, n))
        if np.min(np.diff(a)) > gap:
            return rng.permutation(a)


def fd_grad(f, v, h=1e-6):
    g = np.empty_like(v)
    for i in range(v.shape[0]):
        e = np.zeros_like(v)
        e[i] = h
        g[i] = (f(v + e) - f(v - e)) / (2 * h)
    return g


def test_sym_gradients_match_finite_differences():
    rng = np.random.default_rng(7)
    n, B = 24, 3
    a = separated(rng, n, 0, 6)
    x, g = rng.standard_normal((n, B)), rng.standard_normal((n, B))
    gx, ga = dense.sym_backward(a, x, g)
    np.testing.assert_allclose(ga, fd_grad(lambda t: np.sum(g * dense.sym_apply(t, x)), a), rtol=1e-6, atol=1e-8)
    gx_fd = fd_grad(lambda t: np.sum(g * dense.sym_apply(a, t.reshape(n, B))), x.reshape(-1)).reshape(n, B)
    np.testing.assert_allclose(gx, gx_fd, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("phased", [False, True])
@pytest.mark.parametrize("transpose", [False, True])
def test_rect_gradients_match_finite_differences(phased, transpose):
    rng = np.random.default_rng(8 + 2 * phased + transpose)
    n, k, B = 15, 9, 2
    a, b = separated(rng, n, 0, 5, 1e-3), separated(rng, k, 0.01, 5.01, 1e-3)
    while np.min(np.abs(a[:, None] - b[None, :])) < 1e-3:
        b = separated(rng, k, 0.01, 5.01, 1e-3)
    phi = rng.uniform(0, 2 * np.pi, n) if phased else None
    psi = rng.uniform(0, 2 * np.pi, k) if phased else None
    x = rng.standard_normal(((n if transpose else k), B))
    g = rng.standard_normal(((k if transpose else n), B))
    gr = dense.rect_backward(a, b, x, g, phi, psi, transpose)

    def loss(a_=a, b_=b, phi_=phi, psi_=psi, x_=x):
        return np.sum(g * dense.rect_apply(a_, b_, x_, phi_, psi_, transpose))

    np.testing.assert_allclose(gr["ga"], fd_grad(lambda t: loss(a_=t), a), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(gr["gb"], fd_grad(lambda t: loss(b_=t), b), rtol=1e-6, atol=1e-8)
    shp = x.shape
    np.testing.assert_allclose(gr["gx"], fd_grad(lambda t: loss(x_=t.reshape(shp)), x.reshape(-1)).reshape(shp),
                               rtol=1e-6, atol=1e-8)
    if phased:
        np.testing.assert_allclose(gr["gphi"], fd_grad(lambda t: loss(phi_=t), phi), rtol=1e-6, atol=1e-8)
        np.testing.assert_allclose(gr["gpsi"], fd_grad(lambda t: loss(psi_=t), psi), rtol=1e-6, atol=1e-8)


def test_gram_D_gradient_matches_finite_differences():
    rng = np.random.default_rng(12)
    a, b = rng.uniform(0, 8, 20), rng.uniform(0, 8, 6)
    D = rng.uniform(0.1, 2, 6)
    v, g = rng.standard_normal((20, 2)), rng.standard_normal((20, 2))
    gD = dense.gram_backward_D(a, b, v, g)
    np.testing.assert_allclose(gD, fd_grad(lambda t: np.sum(g * dense.gram_apply(a, b, t, v)), D), rtol=1e-7)


def test_gram_full_backward_matches_finite_differences():
    """gv, ga, gb and gD of <g, A diag(D) A^T v> against central differences of the
    dense forward (anchors kept 1e-3 apart, so no |a_i - b_j| crosses zero)."""
    rng = np.random.default_rng(15)
    n, k, B = 14, 6, 2
    a, b = separated(rng, n, 0, 6, 1e-3), separated(rng, k, 0.01, 6.01, 1e-3)
    while np.min(np.abs(a[:, None] - b[None, :])) < 1e-3:
        b = separated(rng, k, 0.01, 6.01, 1e-3)
    D = rng.uniform(0.1, 2, k)
    v, g = rng.standard_normal((n, B)), rng.standard_normal((n, B))
    gr = dense.gram_backward(a, b, D, v, g)

    def loss(a_=a, b_=b, D_=D, v_=v):
        return np.sum(g * dense.gram_apply(a_, b_, D_, v_))

    np.testing.assert_allclose(gr["ga"], fd_grad(lambda t: loss(a_=t), a), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(gr["gb"], fd_grad(lambda t: loss(b_=t), b), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(gr["gD"], fd_grad(lambda t: loss(D_=t), D), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(gr["gv"], fd_grad(lambda t: loss(v_=t.reshape(v.shape)), v.reshape(-1)).reshape(v.shape),
                               rtol=1e-7, atol=1e-9)
    # the operator is symmetric, so gv is the operator applied to g
    np.testing.assert_allclose(gr["gv"], dense.gram_apply(a, b, D, g), rtol=1e-12)
    # shifting every anchor leaves the loss unchanged (ties included): sum ga + sum gb = 0
    assert abs(gr["ga"].sum() + gr["gb"].sum()) < 1e-10 * (np.abs(gr["ga"]).sum() + np.abs(gr["gb"]).sum())


def test_planted_gram_gradient_mistake_fails_the_fd_pin():
    """A gradient that forgets the dependence of w = A^T v on the anchors (keeping
    only the outer A) is caught by the finite-difference pin."""
    rng = np.random.default_rng(16)
    n, k = 12, 5
    a, b = separated(rng, n, 0, 5, 1e-3), separated(rng, k, 0.01, 5.01, 1e-3)
    while np.min(np.abs(a[:, None] - b[None, :])) < 1e-3:
        b = separated(rng, k, 0.01, 5.01, 1e-3)
    D = rng.uniform(0.1, 2, k)
    v, g = rng.standard_normal((n, 1)), rng.standard_normal((n, 1))
    A, S = dense.kernel(a, b), dense.sign_matrix(a, b)
    w = A.T @ v
    wrong_ga = (-S * A * D[None, :] * (g @ w.T)).sum(axis=1)  # the v u^T term dropped
    fd = fd_grad(lambda t: np.sum(g * dense.gram_apply(t, b, D, v)), a)
    assert not np.allclose(wrong_ga, fd, rtol=1e-4, atol=1e-6)
    np.testing.assert_allclose(dense.gram_backward(a, b, D, v, g)["ga"], fd, rtol=1e-6, atol=1e-8)


def test_gram_is_positive_semidefinite_and_symmetric():
    rng = np.random.default_rng(13)
    a, b = rng.uniform(0, 8, 40), rng.uniform(0, 8, 7)
    D = rng.uniform(0.1, 2, 7)
    M = dense.gram_matrix(a, b, D)
    np.testing.assert_allclose(M, M.T, rtol=1e-14)
    for _ in range(4):
        v = rng.standard_normal(40)
        assert v @ dense.gram_apply(a, b, D, v)[:, 0] >= -1e-12


def test_gradient_invariances_with_ties():
    rng = np.random.default_rng(14)
    a = (rng.integers(0, 12, 30) * 0.5).astype(np.float32)  # many exact ties
    b = (rng.integers(0, 12, 10) * 0.5).astype(np.float32)
    x, g = rng.standard_normal((30, 2)), rng.standard_normal((30, 2))
    _, ga = dense.sym_backward(a, x, g)
    assert abs(ga.sum()) < 1e-12 * np.abs(ga).sum() + 1e-12  # shifting every anchor changes nothing
    phi, psi = rng.uniform(0, 6, 30), rng.uniform(0, 6, 10)
    xb = rng.standard_normal((10, 2))
    gr = dense.rect_backward(a, b, xb, g, phi, psi)
    assert abs(gr["ga"].sum() + gr["gb"].sum()) < 1e-12 * (np.abs(gr["ga"]).sum() + 1)
    assert abs(gr["gphi"].sum() + gr["gpsi"].sum()) < 1e-12 * (np.abs(gr["gphi"]).sum() + 1)


def test_twins_bound_the_outputs():
    rng = np.random.default_rng(15)
    a, b = rng.uniform(0, 5, 25), rng.uniform(0, 5, 8)
    phi, psi = rng.uniform(0, 6, 25), rng.uniform(0, 6, 8)
    x, g = rng.standard_normal((8, 2)), rng.standard_normal((25, 2))
    assert np.all(np.abs(dense.rect_apply(a, b, x, phi, psi)) <= dense.rect_apply(a, b, x, phi, psi, twin=True) + 1e-15)
    gr = dense.rect_backward(a, b, x, g, phi, psi)
    gt = dense.rect_backward(a, b, x, g, phi, psi, twin=True)
    for key in gr:
        assert np.all(np.abs(gr[key]) <= gt[key] + 1e-14), key


# A mistake planted in a copy of the definitions must be caught by the pins above.
def _planted_ga_without_column_term(a, x, g):
    K, S = dense.kernel(a, a), dense.sign_matrix(a, a)
    return (-(S * K * (g @ x.T))).sum(axis=1)


def _planted_ga_flipped_sign(a, x, g):
    return -dense.sym_backward(a, x, g)[1]


@pytest.mark.parametrize("planted", [_planted_ga_without_column_term, _planted_ga_flipped_sign])
def test_planted_gradient_mistakes_fail_the_fd_pin(planted):
    rng = np.random.default_rng(16)
    n = 12
    a = separated(rng, n, 0, 4)
    x, g = rng.standard_normal((n, 2)), rng.standard_normal((n, 2))
    fd = fd_grad(lambda t: np.sum(g * dense.sym_apply(t, x)), a)
    assert not np.allclose(planted(a, x, g), fd, rtol=1e-6, atol=1e-8)


def test_planted_missing_diagonal_fails_the_closed_form():
    n, delta = 50, 0.25
    a = (np.arange(1, n + 1) * delta).astype(np.float32)
    wrong = dense.sym_apply(a, np.ones(n))[:, 0] - 1.0  # diagonal dropped
    assert not np.allclose(wrong, grid_closed_form(n, delta), rtol=1e-6)
