"""Every operator at wide batches, up to the ABI's LAPLEX_MAX_B = 1024, against the
fp64 oracle (elementwise within 1e-5 * twin + 1e-30), with ties inside a, inside b
and between them.

Past 32 channels the symmetric path runs several channel groups whose anchor
gradients add up atomically; past 32 lanes of a row (128 channels in 16-byte
slices, 32 in 4-byte ones) the rectangular large-side pass splits each row into
chunks whose anchor and phase gradients add up atomically.  B = 33 and 129 take the
4-byte slices (B not a multiple of 4), 256 and 1024 the 16-byte ones."""
import numpy as np
import pytest

import oracle
from structured_trainable_laplace_b200 import inputs
from tests.gpu_util import laplex_or_fail
from tests.parity import assert_close
from tests.test_gpu_rect import OPS, compare_gram, compare_gram_backward, compare_rect
from tests.test_gpu_sym import compare

pytestmark = pytest.mark.gpu

WIDE = [33, 129, 256, 1024]


@pytest.fixture(scope="module")
def L():
    return laplex_or_fail()


@pytest.mark.parametrize("B", WIDE)
@pytest.mark.parametrize("saved", [True, False])
def test_sym_wide(L, B, saved):
    n = 3000 if B >= 256 else 9000
    w = inputs.symmetric(n, B, seed=B, tie_frac=0.05)
    compare(L, w["a"], w["x"], w["g"], saved, tag=f"n{n} B{B}")


def _rect_inputs(n, k, B, op, seed, quant):
    rng = np.random.default_rng(seed)
    a, b = rng.uniform(0, 20, n), rng.uniform(0, 20, k)
    if quant:
        a, b = np.round(a / quant) * quant, np.round(b / quant) * quant
    a, b = a.astype(np.float32), b.astype(np.float32)
    phased, transpose = OPS[op]
    x = rng.standard_normal(((n if transpose else k), B)).astype(np.float32)
    g = rng.standard_normal(((k if transpose else n), B)).astype(np.float32)
    phi = rng.uniform(0, 2 * np.pi, n).astype(np.float32)
    psi = rng.uniform(0, 2 * np.pi, k).astype(np.float32)
    return a, b, x, g, phi, psi


@pytest.mark.parametrize("op", list(OPS))
@pytest.mark.parametrize("B", WIDE)
@pytest.mark.parametrize("n,k", [(2000, 300), (300, 2000)])
def test_rect_wide(L, op, B, n, k):
    a, b, x, g, phi, psi = _rect_inputs(n, k, B, op, seed=n + 3 * k + B, quant=0.05)
    compare_rect(L, op, a, b, x, g, phi, psi, saved=(B % 2 == 0), tag=f"n{n} k{k} B{B}")


@pytest.mark.parametrize("op", list(OPS))
@pytest.mark.parametrize("n,k,B", [(300_000, 5000, 64), (5000, 300_000, 64), (200_000, 70_000, 12),
                                   (100_000, 3000, 160)])
def test_rect_large_sides(L, op, n, k, B):
    """Both sides past one tile of the small-side scan, wide lane groups (B = 64,
    160) and narrow ones (B = 12), the large side over many CTAs."""
    a, b, x, g, phi, psi = _rect_inputs(n, k, B, op, seed=n + k + B, quant=0.001)
    compare_rect(L, op, a, b, x, g, phi, psi, saved=True, tag=f"n{n} k{k} B{B}")


@pytest.mark.parametrize("B", WIDE)
@pytest.mark.parametrize("n,k", [(3000, 200), (200, 3000)])
def test_gram_wide(L, B, n, k):
    w = inputs.gram(n, k, B, seed=n + k + B, span=30.0)
    compare_gram(L, w["a"], w["b"], w["D"], w["v"], w["g"], tag=f"n{n} k{k} B{B}")


@pytest.mark.parametrize("B", WIDE)
@pytest.mark.parametrize("n,k", [(2500, 150), (150, 2500)])
def test_gram_backward_wide(L, B, n, k):
    rng = np.random.default_rng(n * 7 + k + B)
    a = (np.round(rng.uniform(0, 25, n) / 0.05) * 0.05).astype(np.float32)
    b = (np.round(rng.uniform(0, 25, k) / 0.05) * 0.05).astype(np.float32)
    D = np.log1p(np.exp(rng.standard_normal(k))).astype(np.float32)
    v = rng.standard_normal((n, B)).astype(np.float32)
    g = rng.standard_normal((n, B)).astype(np.float32)
    compare_gram_backward(L, a, b, D, v, g, oracle.gram_backward, tag=f"n{n} k{k} B{B}")


def test_batch_past_the_limit_is_rejected(L):
    import torch
    a = torch.zeros(16, device="cuda")
    s, p = L.sort_anchors(a)
    x = torch.zeros(16, 1025, device="cuda")
    with pytest.raises(L.LaplexError) as ei:
        L.apply_sym(s, p, x)
    assert ei.value.code == 1
