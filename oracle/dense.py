"""Dense fp64 definitions of the LAPLEX operators (tiny sizes only).

TEST INFRASTRUCTURE ONLY.  Each function writes out a definition from
"LAPLEX: The FFT of Learnable Laplace Kernels" (gist.science technical summary):

* section 2.1, the operator: K_ij = exp(-|a_i - b_j|), and the phased operator
  K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j);
* section 2.2, "Gram operators": M = A diag(D) A^T, applied to v;
* the gradients of the scalar <g, out> with respect to every input, from the
  derivative of each matrix entry:  d/da_i exp(-|a_i - b_j|) = -sign(a_i - b_j) K_ij,
  d/db_j = +sign(a_i - b_j) K_ij, with sign(0) = 0 (the convention of the
  absolute value's derivative used by array libraries), and
  d/dphi_i cos(phi_i - psi_j) = -sin(phi_i - psi_j).

Everything is an explicit n x k matrix, so the cost is O(n k).  ``twin=True``
returns the magnitude companion: every factor replaced by its absolute value.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    # exact promotion of fp32 inputs; fp64 inputs (finite-difference probes) pass unchanged
    return np.asarray(x, dtype=np.float64)


def _rows(x):
    x = _f64(x)
    return x[:, None] if x.ndim == 1 else x


def kernel(a, b):
    """E_ij = exp(-|a_i - b_j|)."""
    a, b = _f64(a), _f64(b)
    return np.exp(-np.abs(a[:, None] - b[None, :]))


def sign_matrix(a, b):
    """S_ij = sign(a_i - b_j), with sign(0) = 0."""
    a, b = _f64(a), _f64(b)
    return np.sign(a[:, None] - b[None, :])


def phase_matrices(phi, psi):
    """(cos(phi_i - psi_j), sin(phi_i - psi_j))."""
    d = _f64(phi)[:, None] - _f64(psi)[None, :]
    return np.cos(d), np.sin(d)


def operator(a, b, phi=None, psi=None):
    """The (phased) LAPLEX matrix."""
    E = kernel(a, b)
    if phi is not None:
        E = E * phase_matrices(phi, psi)[0]
    return E


def sym_apply(a, x, twin=False):
    """y = K x with K = LAPLEX(a, a)."""
    x = _rows(x)
    K = kernel(a, a)
    return K @ (np.abs(x) if twin else x)


def sym_backward(a, x, g, twin=False):
    """Gradients of l = sum_{p,q,c} g_pc K_pq x_qc.

    gx = K^T g.  Anchor a_i enters row i and column i of K:
    dK_pq/da_i = -sign(a_p - a_q) K_pq (delta_pi - delta_qi), so
    ga_i = -sum_q S_iq K_iq M_iq + sum_p S_pi K_pi M_pi with M = g x^T summed over c.
    """
    x, g = _rows(x), _rows(g)
    K = kernel(a, a)
    S = sign_matrix(a, a)
    if twin:
        x, g, S = np.abs(x), np.abs(g), np.abs(S)
        M = g @ x.T
        W = S * K * M
        return K.T @ g, W.sum(axis=1) + W.sum(axis=0)
    M = g @ x.T
    W = S * K * M
    return K.T @ g, -W.sum(axis=1) + W.sum(axis=0)


def rect_apply(a, b, x, phi=None, psi=None, transpose=False, twin=False):
    """y = E x (x at b, y at a), or z = E^T x (x at a, z at b)."""
    x = _rows(x)
    if twin:
        E = kernel(a, b)
        if phi is None:
            A = E
            return (A.T if transpose else A) @ np.abs(x)
        # cos/sin split of cos(phi_i - psi_j), each factor made non-negative
        cp, sp = np.abs(np.cos(_f64(phi))), np.abs(np.sin(_f64(phi)))
        cq, sq = np.abs(np.cos(_f64(psi))), np.abs(np.sin(_f64(psi)))
        ax = np.abs(x)
        if not transpose:
            return cp[:, None] * (E @ (cq[:, None] * ax)) + sp[:, None] * (E @ (sq[:, None] * ax))
        return cq[:, None] * (E.T @ (cp[:, None] * ax)) + sq[:, None] * (E.T @ (sp[:, None] * ax))
    E = operator(a, b, phi, psi)
    return (E.T if transpose else E) @ x


def rect_backward(a, b, x, g, phi=None, psi=None, transpose=False, twin=False):
    """Gradients of l = <g, out> for rect_apply, entry by entry.

    With M_ij = sum_c g_ic x_jc (forward) or sum_c x_ic g_jc (transpose), and
    l = sum_ij W_ij M_ij for W = exp(-|a_i - b_j|) cos(phi_i - psi_j):
      ga_i = sum_j -S_ij W_ij M_ij,   gb_j = sum_i S_ij W_ij M_ij,
      gphi_i = sum_j -E_ij sin(phi_i - psi_j) M_ij,  gpsi_j = sum_i E_ij sin(phi_i - psi_j) M_ij,
      gx = W^T g (forward) or W g (transpose).
    ``twin=True`` gives the magnitude companion of each gradient.
    """
    x, g = _rows(x), _rows(g)
    E = kernel(a, b)
    S = sign_matrix(a, b)
    if phi is not None:
        C, Sn = phase_matrices(phi, psi)
    else:
        C, Sn = np.ones_like(E), np.zeros_like(E)
    if twin:
        # magnitude companion: the cos/sin split with every factor non-negative
        x, g, S = np.abs(x), np.abs(g), np.abs(S)
        if phi is not None:
            cp, sp = np.abs(np.cos(_f64(phi))), np.abs(np.sin(_f64(phi)))
            cq, sq = np.abs(np.cos(_f64(psi))), np.abs(np.sin(_f64(psi)))
            C = cp[:, None] * cq[None, :] + sp[:, None] * sq[None, :]
            Sn = -(sp[:, None] * cq[None, :] + cp[:, None] * sq[None, :])
    W = E * C
    if not transpose:
        M = g @ x.T
        gx = W.T @ g
    else:
        M = x @ g.T
        gx = W @ g
    sg = -1.0 if twin else 1.0
    out = {
        "gx": gx,
        "ga": (sg * -S * W * M).sum(axis=1),
        "gb": (S * W * M).sum(axis=0),
    }
    if phi is not None:
        out["gphi"] = (-E * Sn * M).sum(axis=1)
        out["gpsi"] = (sg * E * Sn * M).sum(axis=0)
    return out


def gram_matrix(a, b, D):
    """M = A diag(D) A^T, A_ij = exp(-|a_i - b_j|)."""
    A = kernel(a, b)
    return (A * _f64(D)[None, :]) @ A.T


def gram_apply(a, b, D, v, twin=False):
    """Sigma v = A diag(D) A^T v."""
    v = _rows(v)
    A = kernel(a, b)
    Dv = _f64(D)
    if twin:
        return A @ (np.abs(Dv)[:, None] * (A.T @ np.abs(v)))
    return A @ (Dv[:, None] * (A.T @ v))


def gram_backward_D(a, b, v, g):
    """d/dD_j <g, A diag(D) A^T v> = sum_c (A^T g)_jc (A^T v)_jc."""
    v, g = _rows(v), _rows(g)
    A = kernel(a, b)
    return ((A.T @ g) * (A.T @ v)).sum(axis=1)


def gram_backward(a, b, D, v, g, twin=False):
    """Every gradient of l = <g, A diag(D) A^T v> (A_ij = exp(-|a_i - b_j|)), entry by
    entry.  With w = A^T v and u = A^T g, l = sum_jc D_j u_jc w_jc, and
    dl/dA_ij = D_j M_ij with M_ij = sum_c (g_ic w_jc + v_ic u_jc); with the entry
    derivatives of the module docstring:
      gv = A (D u) (the operator is symmetric),  gD_j = sum_c u_jc w_jc,
      ga_i = sum_j -S_ij A_ij D_j M_ij,  gb_j = sum_i S_ij A_ij D_j M_ij.
    ``twin=True``: every factor (and w, u) replaced by its magnitude companion."""
    v, g = _rows(v), _rows(g)
    A = kernel(a, b)
    S = sign_matrix(a, b)
    Dv = _f64(D)
    sg = 1.0
    if twin:
        v, g, S, Dv, sg = np.abs(v), np.abs(g), np.abs(S), np.abs(Dv), -1.0
    w, u = A.T @ v, A.T @ g
    M = g @ w.T + v @ u.T
    W = A * Dv[None, :] * M
    return {
        "gv": A @ (Dv[:, None] * u),
        "ga": (sg * -S * W).sum(axis=1),
        "gb": (S * W).sum(axis=0),
        "gD": (u * w).sum(axis=1),
    }

