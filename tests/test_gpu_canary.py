"""Out-of-bounds writes, without a sanitizer: every output, saved buffer and
workspace is placed inside a larger device allocation whose guard regions hold a
canary bit pattern, at odd and ragged sizes, and every call must leave the guards
intact.  Inputs get guards too, which must never be read into the results (the
results are compared with the oracle)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import laplex_or_fail
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes of guard on each side (a multiple of 16: keeps 16-byte alignment)
CANARY = 0x7fc0dead   # a NaN bit pattern


@pytest.fixture(scope="module")
def L():
    return laplex_or_fail()


class Guarded:
    """A device buffer of `nbytes` between two canary guards."""

    def __init__(self, nbytes, fill=None):
        self.nbytes = int(nbytes)
        words = (2 * GUARD + ((self.nbytes + 15) // 16) * 16) // 4
        self.raw = torch.full((words,), CANARY, dtype=torch.int32, device="cuda")
        if fill is not None:
            b = np.ascontiguousarray(fill).view(np.uint8).reshape(-1)
            assert b.size == self.nbytes
            self.raw.view(torch.uint8)[GUARD:GUARD + self.nbytes].copy_(torch.from_numpy(b).cuda())

    @property
    def ptr(self):
        return ctypes.c_void_p(self.raw.data_ptr() + GUARD)

    def host(self, dtype, shape):
        b = self.raw.view(torch.uint8)[GUARD:GUARD + self.nbytes].cpu().numpy()
        return b.view(dtype).reshape(shape)

    def intact(self):
        words = self.raw.cpu().numpy()
        g = GUARD // 4
        tail0 = (GUARD + ((self.nbytes + 15) // 16) * 16) // 4
        # the padding between nbytes and the next 16-byte boundary is not a guard
        return bool(np.all(words[:g] == CANARY) and np.all(words[tail0:] == CANARY))


def status(L):
    st = Guarded(4, np.zeros(1, np.int32))
    return st


def read_status(L, st):
    h = ctypes.c_int32(0)
    code = L.lib().laplex_read_status(st.ptr, None, ctypes.byref(h))
    return code


@pytest.mark.parametrize("n,B", [(1, 1), (4097, 1), (515, 3), (70001, 16), (3000, 33)])
def test_sym_forward_backward_stay_in_bounds(L, n, B):
    lib = L.lib()
    rng = np.random.default_rng(n + B)
    a = rng.uniform(0, 0.05 * n + 1, n).astype(np.float32)
    a[rng.choice(n, size=n // 20, replace=False)] = a[0]  # ties
    x = rng.standard_normal((n, B)).astype(np.float32)
    g = rng.standard_normal((n, B)).astype(np.float32)
    A, X, G = Guarded(4 * n, a), Guarded(4 * n * B, x), Guarded(4 * n * B, g)
    S, P = Guarded(4 * n), Guarded(4 * n)
    Y, GX, GA = Guarded(4 * n * B), Guarded(4 * n * B), Guarded(4 * n)
    sws = Guarded(lib.laplex_sort_workspace_size(n))
    ws = Guarded(lib.laplex_workspace_size(0, n, 1, B))
    sv = Guarded(lib.laplex_saved_size(0, n, 1, B))
    st = status(L)
    assert lib.laplex_sort_anchors(A.ptr, n, S.ptr, P.ptr, sws.ptr, sws.nbytes, st.ptr, None) == 0
    assert lib.laplex_apply_sym(S.ptr, P.ptr, n, X.ptr, B, Y.ptr, sv.ptr, ws.ptr, ws.nbytes, st.ptr, None) == 0
    assert lib.laplex_backward(0, S.ptr, P.ptr, n, None, None, None, 1, None, X.ptr, G.ptr, B, sv.ptr, GX.ptr,
                               GA.ptr, None, None, None, ws.ptr, ws.nbytes, st.ptr, None) == 0
    assert read_status(L, st) == 0
    for name, buf in [("a", A), ("x", X), ("g", G), ("a_sorted", S), ("perm", P), ("y", Y), ("gx", GX),
                      ("ga", GA), ("sort ws", sws), ("ws", ws), ("saved", sv), ("status", st)]:
        assert buf.intact(), f"{name}: guard overwritten (n={n}, B={B})"
    assert_close(Y.host(np.float32, (n, B)), oracle.sym_apply(a, x), oracle.sym_apply(a, x, twin=True), "y")
    gx_ref, ga_ref = oracle.sym_backward(a, x, g)
    gx_tw, ga_tw = oracle.sym_backward(a, x, g, twin=True)
    assert_close(GX.host(np.float32, (n, B)), gx_ref, gx_tw, "gx")
    assert_close(GA.host(np.float32, (n,)), ga_ref, ga_tw, "ga")


@pytest.mark.parametrize("n,k,B,transpose", [(5003, 129, 3, True), (129, 5003, 5, False), (70000, 1000, 8, True),
                                             (2000, 2000, 128, True)])
def test_phased_forward_backward_stay_in_bounds(L, n, k, B, transpose):
    lib = L.lib()
    rng = np.random.default_rng(n * 3 + k)
    a = rng.uniform(0, 30, n).astype(np.float32)
    b = rng.uniform(0, 30, k).astype(np.float32)
    phi = rng.uniform(0, 2 * np.pi, n).astype(np.float32)
    psi = rng.uniform(0, 2 * np.pi, k).astype(np.float32)
    rows_in, rows_out = (n, k) if transpose else (k, n)
    x = rng.standard_normal((rows_in, B)).astype(np.float32)
    g = rng.standard_normal((rows_out, B)).astype(np.float32)
    op = 4 if transpose else 3
    A, Bb, PH, PS = Guarded(4 * n, a), Guarded(4 * k, b), Guarded(4 * n, phi), Guarded(4 * k, psi)
    X, G = Guarded(4 * rows_in * B, x), Guarded(4 * rows_out * B, g)
    SA, PA, SB, PB = Guarded(4 * n), Guarded(4 * n), Guarded(4 * k), Guarded(4 * k)
    OUT, GX = Guarded(4 * rows_out * B), Guarded(4 * rows_in * B)
    GA, GB, GPHI, GPSI = Guarded(4 * n), Guarded(4 * k), Guarded(4 * n), Guarded(4 * k)
    sws = Guarded(lib.laplex_sort_workspace_size(max(n, k)))
    ws = Guarded(lib.laplex_workspace_size(op, n, k, B))
    sv = Guarded(lib.laplex_saved_size(op, n, k, B))
    st = status(L)
    assert lib.laplex_sort_anchors(A.ptr, n, SA.ptr, PA.ptr, sws.ptr, sws.nbytes, st.ptr, None) == 0
    assert lib.laplex_sort_anchors(Bb.ptr, k, SB.ptr, PB.ptr, sws.ptr, sws.nbytes, st.ptr, None) == 0
    assert lib.laplex_apply_phased(SA.ptr, PA.ptr, n, PH.ptr, SB.ptr, PB.ptr, k, PS.ptr, int(transpose), X.ptr, B,
                                   OUT.ptr, sv.ptr, ws.ptr, ws.nbytes, st.ptr, None) == 0
    assert lib.laplex_backward(op, SA.ptr, PA.ptr, n, PH.ptr, SB.ptr, PB.ptr, k, PS.ptr, X.ptr, G.ptr, B, sv.ptr,
                               GX.ptr, GA.ptr, GB.ptr, GPHI.ptr, GPSI.ptr, ws.ptr, ws.nbytes, st.ptr, None) == 0
    assert read_status(L, st) == 0
    for name, buf in [("out", OUT), ("gx", GX), ("ga", GA), ("gb", GB), ("gphi", GPHI), ("gpsi", GPSI),
                      ("ws", ws), ("saved", sv), ("sort ws", sws), ("x", X), ("g", G)]:
        assert buf.intact(), f"{name}: guard overwritten (n={n}, k={k}, B={B}, transpose={transpose})"
    ref = oracle.rect_apply(a, b, x, phi, psi, transpose)
    assert_close(OUT.host(np.float32, ref.shape), ref, oracle.rect_apply(a, b, x, phi, psi, transpose, twin=True),
                 "out")
    grads = oracle.rect_backward(a, b, x, g, phi, psi, transpose)
    twins = oracle.rect_backward(a, b, x, g, phi, psi, transpose, twin=True)
    got = {"gx": GX.host(np.float32, x.shape), "ga": GA.host(np.float32, (n,)), "gb": GB.host(np.float32, (k,)),
           "gphi": GPHI.host(np.float32, (n,)), "gpsi": GPSI.host(np.float32, (k,))}
    for key in grads:
        assert_close(got[key], grads[key], twins[key], key)


@pytest.mark.parametrize("n,k,B", [(9001, 513, 4), (300, 3000, 3)])
def test_gram_stays_in_bounds(L, n, k, B):
    lib = L.lib()
    rng = np.random.default_rng(n + 7 * k)
    a = rng.uniform(0, 40, n).astype(np.float32)
    b = rng.uniform(0, 40, k).astype(np.float32)
    D = np.log1p(np.exp(rng.standard_normal(k))).astype(np.float32)
    v = rng.standard_normal((n, B)).astype(np.float32)
    g = rng.standard_normal((n, B)).astype(np.float32)
    A, Bb, DD, V, G = Guarded(4 * n, a), Guarded(4 * k, b), Guarded(4 * k, D), Guarded(4 * n * B, v), \
        Guarded(4 * n * B, g)
    SA, PA, SB, PB = Guarded(4 * n), Guarded(4 * n), Guarded(4 * k), Guarded(4 * k)
    Y, W, GD = Guarded(4 * n * B), Guarded(4 * k * B), Guarded(4 * k)
    sws = Guarded(lib.laplex_sort_workspace_size(max(n, k)))
    ws = Guarded(lib.laplex_workspace_size(5, n, k, B))
    st = status(L)
    assert lib.laplex_sort_anchors(A.ptr, n, SA.ptr, PA.ptr, sws.ptr, sws.nbytes, st.ptr, None) == 0
    assert lib.laplex_sort_anchors(Bb.ptr, k, SB.ptr, PB.ptr, sws.ptr, sws.nbytes, st.ptr, None) == 0
    assert lib.laplex_gram_apply(SA.ptr, PA.ptr, n, SB.ptr, PB.ptr, k, DD.ptr, V.ptr, B, Y.ptr, W.ptr, G.ptr, GD.ptr,
                                 ws.ptr, ws.nbytes, st.ptr, None) == 0
    assert read_status(L, st) == 0
    for name, buf in [("y", Y), ("w", W), ("gD", GD), ("ws", ws), ("sort ws", sws)]:
        assert buf.intact(), f"{name}: guard overwritten (n={n}, k={k}, B={B})"
    assert_close(Y.host(np.float32, (n, B)), oracle.gram_apply(a, b, D, v), oracle.gram_apply(a, b, D, v, twin=True),
                 "gram y")
    assert_close(GD.host(np.float32, (k,)), oracle.gram_backward_D(a, b, v, g),
                 oracle.gram_backward_D(a, b, v, g, twin=True), "gram gD")
