"""Stream use of the binding.  Every entry point is stream-ordered and never
synchronises, so a whole training step (sort, forward, backward) can be captured
once as a CUDA graph and replayed on new inputs copied into the captured input
buffers; the replays must match the fp64 oracle on those new inputs like the eager
calls do.  Calls on two streams at once use separate scratch and must each match."""
import numpy as np
import pytest

import oracle
from structured_trainable_laplace_b200 import inputs
from tests.gpu_util import dev, host, laplex_or_fail
from tests.parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    return laplex_or_fail()


def capture(torch, step, warm=2):
    """Run `step` on a side stream (workspaces reach full size), then capture it."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warm):
            step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = step()
    return g, out


@pytest.mark.parametrize("n,B", [(4096, 1), (30_011, 16), (100_003, 1)])
def test_symmetric_train_step_replays(L, n, B):
    import torch
    w0 = inputs.symmetric(n, B, seed=31, tie_frac=0.05)
    t = {k: dev(v) for k, v in w0.arrays.items()}
    saved = L.saved_buffer("sym", n, 1, B, t["a"].device)

    def step():
        s, p = L.sort_anchors(t["a"])
        y = L.apply_sym(s, p, t["x"], saved=saved)
        gr = L.backward("sym", s, p, t["x"], t["g"], saved=saved, need=("gx", "ga"))
        return y, gr["gx"], gr["ga"]

    g, (y, gx, ga) = capture(torch, step)
    for seed in (32, 33):  # new anchors (new sort) and vectors in the captured buffers
        w = inputs.symmetric(n, B, seed=seed, tie_frac=0.05)
        for k, v in w.arrays.items():
            t[k].copy_(dev(v))
        g.replay()
        torch.cuda.synchronize()
        L.check()
        a, x, gg = w["a"], w["x"], w["g"]
        assert_close(host(y).reshape(n, B), oracle.sym_apply(a, x), oracle.sym_apply(a, x, twin=True), "y")
        gx_ref, ga_ref = oracle.sym_backward(a, x, gg)
        gx_tw, ga_tw = oracle.sym_backward(a, x, gg, twin=True)
        assert_close(host(gx).reshape(n, B), gx_ref, gx_tw, "gx")
        assert_close(host(ga), ga_ref, ga_tw, "ga")
    del g


def test_phased_head_train_step_replays(L):
    import torch
    n, k, B = 20_000, 300, 8
    w0 = inputs.phased_head(n, k, B, seed=41)
    t = {key: dev(v) for key, v in w0.arrays.items()}
    saved = L.saved_buffer("phased_transpose", n, k, B, t["a"].device)

    def step():
        sa, pa = L.sort_anchors(t["a"])
        sb, pb = L.sort_anchors(t["b"])
        z = L.apply_phased(sa, pa, t["phi"], sb, pb, t["psi"], t["x"], transpose=True, saved=saved)
        gr = L.backward("phased_transpose", sa, pa, t["x"], t["h"], b_sorted=sb, perm_b=pb, phi=t["phi"],
                        psi=t["psi"], saved=saved)
        return z, gr

    g, (z, gr) = capture(torch, step)
    w = inputs.phased_head(n, k, B, seed=42)
    for key, v in w.arrays.items():
        t[key].copy_(dev(v))
    g.replay()
    torch.cuda.synchronize()
    L.check()
    a, b, phi, psi, x, h = w["a"], w["b"], w["phi"], w["psi"], w["x"], w["h"]
    assert_close(host(z).reshape(k, B), oracle.rect_apply(a, b, x, phi, psi, transpose=True),
                 oracle.rect_apply(a, b, x, phi, psi, transpose=True, twin=True), "z")
    ref = oracle.rect_backward(a, b, x, h, phi, psi, transpose=True)
    tw = oracle.rect_backward(a, b, x, h, phi, psi, transpose=True, twin=True)
    for key in ("gx", "ga", "gb", "gphi", "gpsi"):
        assert_close(host(gr[key]).reshape(np.shape(ref[key])), ref[key], tw[key], key)
    del g


def test_two_streams_run_concurrently(L):
    # each stream gets its own scratch: interleaved calls on two streams must each
    # match the oracle
    import torch
    ws = [inputs.symmetric(200_003, 4, seed=51), inputs.symmetric(150_001, 8, seed=52)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    dv = [{k: dev(v) for k, v in w.arrays.items()} for w in ws]
    torch.cuda.synchronize()
    outs = [None, None]
    for rep in range(3):
        for i in (0, 1):
            with torch.cuda.stream(streams[i]):
                s, p = L.sort_anchors(dv[i]["a"])
                y = L.apply_sym(s, p, dv[i]["x"])
                gr = L.backward("sym", s, p, dv[i]["x"], dv[i]["g"], need=("gx", "ga"))
                outs[i] = (y, gr["gx"], gr["ga"])
    torch.cuda.synchronize()
    L.check()
    for i, w in enumerate(ws):
        a, x, g = w["a"], w["x"], w["g"]
        y, gx, ga = outs[i]
        assert_close(host(y), oracle.sym_apply(a, x), oracle.sym_apply(a, x, twin=True), f"y{i}")
        gx_ref, ga_ref = oracle.sym_backward(a, x, g)
        gx_tw, ga_tw = oracle.sym_backward(a, x, g, twin=True)
        assert_close(host(gx), gx_ref, gx_tw, f"gx{i}")
        assert_close(host(ga), ga_ref, ga_tw, f"ga{i}")
