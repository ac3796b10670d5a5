"""Rectangular, transposed and phased operators and the Gram apply on the GPU
against the fp64 oracle (forward and every gradient), elementwise within
1e-5 * twin + 1e-30."""
import numpy as np
import pytest

import oracle
from structured_trainable_laplace_b200 import inputs
from tests.gpu_util import dev, host, laplex_or_fail
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

OPS = {"general": (False, False), "transpose": (False, True), "phased": (True, False),
       "phased_transpose": (True, True)}


@pytest.fixture(scope="module")
def L():
    return laplex_or_fail()


def draw(n, k, B, seed, quant=None, span=20.0):
    rng = np.random.default_rng(seed)
    a = rng.uniform(0, span, n)
    b = rng.uniform(0, span, k)
    if quant:  # a coarse grid makes ties inside a, inside b and between a and b
        a, b = np.round(a / quant) * quant, np.round(b / quant) * quant
    return a.astype(np.float32), b.astype(np.float32), rng


def run_rect(L, op, a, b, x, g, phi, psi, saved):
    phased, transpose = OPS[op]
    n, k, B = a.size, b.size, x.shape[1]
    sa, pa = L.sort_anchors(dev(a))
    sb, pb = L.sort_anchors(dev(b))
    sv = L.saved_buffer(op, n, k, B, "cuda") if saved else None
    xt, gt = dev(x), dev(g)
    ph, ps = (dev(phi), dev(psi)) if phased else (None, None)
    if op == "general":
        out = L.apply_general(sa, pa, sb, pb, xt, saved=sv)
    elif op == "transpose":
        out = L.apply_transpose(sa, pa, sb, pb, xt, saved=sv)
    else:
        out = L.apply_phased(sa, pa, ph, sb, pb, ps, xt, transpose=transpose, saved=sv)
    gr = L.backward(op, sa, pa, xt, gt, b_sorted=sb, perm_b=pb, phi=ph, psi=ps, saved=sv)
    L.check()
    return host(out), {key: host(v) for key, v in gr.items()}


def compare_rect(L, op, a, b, x, g, phi=None, psi=None, saved=True, tag=""):
    phased, transpose = OPS[op]
    if not phased:
        phi = psi = None
    out, gr = run_rect(L, op, a, b, x, g, phi, psi, saved)
    assert_close(out, oracle.rect_apply(a, b, x, phi, psi, transpose),
                 oracle.rect_apply(a, b, x, phi, psi, transpose, twin=True), f"{op} out {tag}")
    ref = oracle.rect_backward(a, b, x, g, phi, psi, transpose)
    tw = oracle.rect_backward(a, b, x, g, phi, psi, transpose, twin=True)
    for key in ref:
        assert_close(gr[key], ref[key], tw[key], f"{op} {key} {tag}")


@pytest.mark.parametrize("op", list(OPS))
@pytest.mark.parametrize("n,k,B,quant", [(5000, 300, 3, None), (300, 5000, 4, None), (2000, 2000, 8, 0.05),
                                         (1, 7, 1, None), (7, 1, 2, None), (20000, 1024, 32, 0.01),
                                         (4097, 33, 6, 0.25), (999, 1000, 40, None)])
@pytest.mark.parametrize("saved", [True, False])
def test_rect_ops(L, op, n, k, B, quant, saved):
    a, b, rng = draw(n, k, B, seed=n * 7 + k + B, quant=quant)
    phased, transpose = OPS[op]
    x = rng.standard_normal(((n if transpose else k), B)).astype(np.float32)
    g = rng.standard_normal(((k if transpose else n), B)).astype(np.float32)
    phi = rng.uniform(0, 2 * np.pi, n).astype(np.float32)
    psi = rng.uniform(0, 2 * np.pi, k).astype(np.float32)
    compare_rect(L, op, a, b, x, g, phi, psi, saved, tag=f"n{n} k{k} B{B} q{quant} saved{saved}")


@pytest.mark.parametrize("op", ["general", "phased_transpose"])
def test_rect_small_side_past_direct_tiles(L, op):
    """A small side of more than 1024 scan tiles (600 000 rows, 16 scan channels:
    B = 16, or B = 8 phased: 2344 tiles), so that its scans take the
    decoupled-lookback kernels instead of the totals-then-apply pair."""
    phased, transpose = OPS[op]
    B = 8 if phased else 16
    n, k = 600_000, 600_011
    a, b, rng = draw(n, k, B, seed=77, quant=0.002, span=2000.0)
    x = rng.standard_normal(((n if transpose else k), B)).astype(np.float32)
    g = rng.standard_normal(((k if transpose else n), B)).astype(np.float32)
    phi = rng.uniform(0, 2 * np.pi, n).astype(np.float32)
    psi = rng.uniform(0, 2 * np.pi, k).astype(np.float32)
    compare_rect(L, op, a, b, x, g, phi, psi, saved=True, tag=f"n{n} k{k} B{B}")


def test_phased_head_full_size(L):
    """n = 2^22 -> k = 1024 phased head, B = 128, forward and all five gradients."""
    w = inputs.phased_head_2p22(0)
    compare_rect(L, "phased_transpose", w["a"], w["b"], w["x"], w["h"], w["phi"], w["psi"], tag="head 2^22")


def run_gram(L, a, b, D, v, g):
    sa, pa = L.sort_anchors(dev(a))
    sb, pb = L.sort_anchors(dev(b))
    y, w, gD = L.gram_apply(sa, pa, sb, pb, dev(D), dev(v), g=dev(g), return_w=True)
    L.check()
    return host(y), host(w), host(gD)


def compare_gram(L, a, b, D, v, g, tag=""):
    y, w, gD = run_gram(L, a, b, D, v, g)
    y_ref, w_ref = oracle.gram_apply(a, b, D, v, return_w=True)
    assert_close(y, y_ref, oracle.gram_apply(a, b, D, v, twin=True), f"gram y {tag}")
    assert_close(w, w_ref, oracle.rect_apply(a, b, v, transpose=True, twin=True), f"gram w {tag}")
    assert_close(gD, oracle.gram_backward_D(a, b, v, g), oracle.gram_backward_D(a, b, v, g, twin=True),
                 f"gram gD {tag}")


@pytest.mark.parametrize("n,k,B", [(5000, 200, 3), (200, 5000, 2), (3000, 3000, 8), (1, 1, 1), (9000, 700, 4),
                                   (6000, 500, 6), (7001, 64, 16)])
def test_gram_small(L, n, k, B):
    # n > k takes the paired reduce pass (A^T v and A^T g together, 2B channels)
    w = inputs.gram(n, k, B, seed=n + k, span=30.0)
    compare_gram(L, w["a"], w["b"], w["D"], w["v"], w["g"], tag=f"n{n} k{k}")


@pytest.mark.parametrize("n,k,B", [(5000, 200, 3), (300, 4000, 8)])
def test_gram_without_gradient(L, n, k, B):
    w = inputs.gram(n, k, B, seed=n * 3 + k, span=30.0)
    sa, pa = L.sort_anchors(dev(w["a"]))
    sb, pb = L.sort_anchors(dev(w["b"]))
    y, wv = L.gram_apply(sa, pa, sb, pb, dev(w["D"]), dev(w["v"]), return_w=True)
    L.check()
    y_ref, w_ref = oracle.gram_apply(w["a"], w["b"], w["D"], w["v"], return_w=True)
    assert_close(host(y), y_ref, oracle.gram_apply(w["a"], w["b"], w["D"], w["v"], twin=True), "gram y (no g)")
    assert_close(host(wv), w_ref, oracle.rect_apply(w["a"], w["b"], w["v"], transpose=True, twin=True),
                 "gram w (no g)")


def test_gram_full_size(L):
    """Flattened 3x1024x1024 image: n = 3,145,728, k = 65,536, B = 8."""
    w = inputs.gram_image(0)
    compare_gram(L, w["a"], w["b"], w["D"], w["v"], w["g"], tag="image")


def compare_gram_backward(L, a, b, D, v, g, ref_fn, tag=""):
    sa, pa = L.sort_anchors(dev(a))
    sb, pb = L.sort_anchors(dev(b))
    got = L.gram_backward(sa, pa, sb, pb, dev(D), dev(v), dev(g))
    L.check()
    ref, tw = ref_fn(a, b, D, v, g), ref_fn(a, b, D, v, g, twin=True)
    for key in ("gv", "ga", "gb", "gD"):
        assert_close(host(got[key]), ref[key], tw[key], f"gram {key} {tag}")


@pytest.mark.parametrize("n,k,B,quant", [(4000, 150, 3, None), (150, 4000, 2, None), (2000, 2000, 4, 0.05),
                                         (1, 1, 1, None), (6001, 64, 16, 0.02), (777, 900, 8, 0.25)])
def test_gram_full_backward_small(L, n, k, B, quant):
    """gv, ga, gb, gD of <g, A diag(D) A^T v> against the dense definition (ties
    inside a, inside b and between them when quantised)."""
    rng = np.random.default_rng(n * 5 + k + B)
    a, b = rng.uniform(0, 25, n), rng.uniform(0, 25, k)
    if quant:
        a, b = np.round(a / quant) * quant, np.round(b / quant) * quant
    a, b = a.astype(np.float32), b.astype(np.float32)
    D = np.log1p(np.exp(rng.standard_normal(k))).astype(np.float32)
    v = rng.standard_normal((n, B)).astype(np.float32)
    g = rng.standard_normal((n, B)).astype(np.float32)
    compare_gram_backward(L, a, b, D, v, g, oracle.dense.gram_backward, tag=f"n{n} k{k} B{B} q{quant}")


def test_gram_full_backward_image(L):
    """Flattened 3x1024x1024 image: every gradient against the composed C oracle."""
    w = inputs.gram_image(0)
    compare_gram_backward(L, w["a"], w["b"], w["D"], w["v"], w["g"], oracle.gram_backward, tag="image")
