"""LAPLEX oracle: plain, slow, obviously correct fp64 CPU implementations.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline leg may import this package; the product path never does.

Two independent implementations of what the operators compute:

* ``oracle.dense`` -- the definitions written out with dense fp64 NumPy matrices
  (tiny sizes only): K_ij = exp(-|a_i - b_j|) [cos(phi_i - psi_j)], the Gram
  product A diag(D) A^T v, and the gradients of <g, out> from the derivative of
  each matrix entry, with sign(0) = 0.
* the C library ``laplex_oracle.c`` (wrapped here) -- fp64 sequential sums over
  the distinct values of the merged sorted anchor sequence (strict-left, tie,
  strict-right), usable up to the full workload sizes.

Neither shares code with the CUDA path.  Sort ties follow (value, original
index); -0.0 equals +0.0.  Outputs are fp64 NumPy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import dense  # noqa: F401  (re-exported)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "laplex_oracle.c")
_LIB = os.path.join(_HERE, "liblaplex_oracle.so")

_ERRORS = {1: "bad argument", 4: "non-finite anchor", 7: "out of memory"}


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/liblaplex_oracle.so (gcc, -O2, OpenMP for the
    optional threading of the sampled evaluation)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        D = ctypes.c_double
        lib.oracle_sort.argtypes = [P, I64, P, P]
        lib.oracle_sym_apply.argtypes = [P, I64, P, I64, P, I]
        lib.oracle_sym_backward.argtypes = [P, I64, P, P, I64, P, P, I]
        lib.oracle_rect_apply.argtypes = [P, I64, P, I64, P, P, P, I64, I, P, I]
        lib.oracle_rect_backward.argtypes = [P, I64, P, I64, P, P, P, P, I64, I, P, P, P, P, P, I]
        lib.oracle_gram_apply.argtypes = [P, I64, P, I64, P, P, I64, P, P, I]
        lib.oracle_gram_backward_D.argtypes = [P, I64, P, I64, P, P, I64, P, I]
        lib.oracle_sym_sampled.argtypes = [P, I64, P, P, I64, P, I64, D, P, P, P, P, P, I]
        for f in ("oracle_sort", "oracle_sym_apply", "oracle_sym_backward", "oracle_rect_apply",
                  "oracle_rect_backward", "oracle_gram_apply", "oracle_gram_backward_D", "oracle_sym_sampled"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: {_ERRORS.get(rc, rc)}")


def _rows(x):
    x = _f32(x)
    if x.ndim == 1:
        x = x[:, None]
    return x


def sort(a):
    """Stable sort of the anchors by (value, index).  Returns (a_sorted f32, perm u32)."""
    a = _f32(a)
    n = a.shape[0]
    s = np.empty(n, np.float32)
    p = np.empty(n, np.uint32)
    _check(_load().oracle_sort(_ptr(a), n, _ptr(s), _ptr(p)), "sort")
    return s, p


def sym_apply(a, x, twin=False):
    """y = K x, K_ij = exp(-|a_i - a_j|); x [n][B] -> y [n][B] fp64."""
    a, x = _f32(a), _rows(x)
    n, B = x.shape
    y = np.empty((n, B), np.float64)
    _check(_load().oracle_sym_apply(_ptr(a), n, _ptr(x), B, _ptr(y), int(twin)), "sym_apply")
    return y


def sym_backward(a, x, g, twin=False):
    """Gradients of <g, K x>: returns (gx [n][B], ga [n])."""
    a, x, g = _f32(a), _rows(x), _rows(g)
    n, B = x.shape
    gx = np.empty((n, B), np.float64)
    ga = np.empty(n, np.float64)
    _check(_load().oracle_sym_backward(_ptr(a), n, _ptr(x), _ptr(g), B, _ptr(gx), _ptr(ga), int(twin)),
           "sym_backward")
    return gx, ga


def rect_apply(a, b, x, phi=None, psi=None, transpose=False, twin=False):
    """y = E x (x at b, y at a) or, with transpose, z = E^T x (x at a, z at b).
    E_ij = exp(-|a_i - b_j|) [cos(phi_i - psi_j)]."""
    a, b, x = _f32(a), _f32(b), _rows(x)
    phi = None if phi is None else _f32(phi)
    psi = None if psi is None else _f32(psi)
    n, k = a.shape[0], b.shape[0]
    B = x.shape[1]
    out = np.empty(((k if transpose else n), B), np.float64)
    _check(_load().oracle_rect_apply(_ptr(a), n, _ptr(b), k, _ptr(phi), _ptr(psi), _ptr(x), B, int(transpose),
                                     _ptr(out), int(twin)), "rect_apply")
    return out


def rect_backward(a, b, x, g, phi=None, psi=None, transpose=False, twin=False):
    """Gradients of <g, out> for rect_apply.  Returns dict gx, ga, gb (+ gphi, gpsi if phased)."""
    a, b, x, g = _f32(a), _f32(b), _rows(x), _rows(g)
    phi = None if phi is None else _f32(phi)
    psi = None if psi is None else _f32(psi)
    n, k = a.shape[0], b.shape[0]
    B = x.shape[1]
    gx = np.empty(x.shape, np.float64)
    ga = np.empty(n, np.float64)
    gb = np.empty(k, np.float64)
    gphi = np.empty(n, np.float64) if phi is not None else None
    gpsi = np.empty(k, np.float64) if psi is not None else None
    _check(_load().oracle_rect_backward(_ptr(a), n, _ptr(b), k, _ptr(phi), _ptr(psi), _ptr(x), _ptr(g), B,
                                        int(transpose), _ptr(gx), _ptr(ga), _ptr(gb), _ptr(gphi), _ptr(gpsi),
                                        int(twin)), "rect_backward")
    out = {"gx": gx, "ga": ga, "gb": gb}
    if phi is not None:
        out["gphi"] = gphi
        out["gpsi"] = gpsi
    return out


def gram_apply(a, b, D, v, twin=False, return_w=False):
    """y = A diag(D) A^T v, A_ij = exp(-|a_i - b_j|); v [n][B].  Optionally also w = A^T v."""
    a, b, D, v = _f32(a), _f32(b), _f32(D), _rows(v)
    n, k = a.shape[0], b.shape[0]
    B = v.shape[1]
    y = np.empty((n, B), np.float64)
    w = np.empty((k, B), np.float64) if return_w else None
    _check(_load().oracle_gram_apply(_ptr(a), n, _ptr(b), k, _ptr(D), _ptr(v), B, _ptr(y), _ptr(w), int(twin)),
           "gram_apply")
    return (y, w) if return_w else y


def gram_backward_D(a, b, v, g, twin=False):
    """gD_j = sum_c (A^T g)_j (A^T v)_j."""
    a, b, v, g = _f32(a), _f32(b), _rows(v), _rows(g)
    n, k = a.shape[0], b.shape[0]
    B = v.shape[1]
    gD = np.empty(k, np.float64)
    _check(_load().oracle_gram_backward_D(_ptr(a), n, _ptr(b), k, _ptr(v), _ptr(g), B, _ptr(gD), int(twin)),
           "gram_backward_D")
    return gD


def gram_backward(a, b, D, v, g, twin=False):
    """Every gradient of <g, A diag(D) A^T v>, from the C scans: with w = A^T v and
    u = A^T g (transposed products), gv = A (D u) (a general product), gD = sum_c u w,
    and ga, gb the anchor gradients of the two general products A (D w) read by g
    and A (D u) read by v (dl/dA_ij = D_j sum_c (g_ic w_jc + v_ic u_jc)).
    Returns dict gv, ga, gb, gD (fp64).  ``twin=True`` composes the companions."""
    D = _f32(D).astype(np.float64)
    w = rect_apply(a, b, v, transpose=True, twin=twin)
    u = rect_apply(a, b, g, transpose=True, twin=twin)
    Dm = np.abs(D) if twin else D
    x1, x2 = Dm[:, None] * w, Dm[:, None] * u
    r1 = rect_backward(a, b, x1, g, twin=twin)
    r2 = rect_backward(a, b, x2, v, twin=twin)
    return {
        "gv": rect_apply(a, b, x2, twin=twin),
        "ga": r1["ga"] + r2["ga"],
        "gb": r1["gb"] + r2["gb"],
        "gD": (u * w).sum(axis=1),
    }


def sym_sampled(a, x, samples, g=None, window=100.0, threads=1):
    """Windowed direct evaluation of the symmetric operator at sample indices.
    Returns dict y, y_twin [m][B], dropped [B] (and ga, ga_twin [m] if g given).
    threads > 1 evaluates the samples on that many host threads."""
    a, x = _f32(a), _rows(x)
    g = None if g is None else _rows(g)
    samples = np.ascontiguousarray(samples, dtype=np.int64)
    n, B = x.shape
    m = samples.shape[0]
    y = np.empty((m, B), np.float64)
    yt = np.empty((m, B), np.float64)
    drop = np.empty(B, np.float64)
    ga = np.empty(m, np.float64) if g is not None else None
    gat = np.empty(m, np.float64) if g is not None else None
    _check(_load().oracle_sym_sampled(_ptr(a), n, _ptr(x), _ptr(g), B, _ptr(samples), m, float(window), _ptr(y),
                                      _ptr(yt), _ptr(ga), _ptr(gat), _ptr(drop), int(threads)), "sym_sampled")
    out = {"y": y, "y_twin": yt, "dropped": drop}
    if g is not None:
        out["ga"] = ga
        out["ga_twin"] = gat
    return out
