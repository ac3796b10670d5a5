"""Failure detection on the GPU without a fault: every lookback wait in the
library is bounded, and a wait that runs out records LAPLEX_ERR_TIMEOUT in the
status word and lets its kernel finish.  The self-check entry point runs the
small-side scan's lookback against a predecessor flag that nothing ever sets; the
test checks the recorded status and that the context still computes correctly
afterwards.  Argument errors are checked before any launch (test_abi_cpu)."""
import time

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


def test_unpublished_predecessor_times_out_and_the_context_survives(L):
    t0 = time.perf_counter()
    code = L.check_wait_bound()
    elapsed = time.perf_counter() - t0
    assert code == 5, f"expected LAPLEX_ERR_TIMEOUT (5), got {code}"
    assert elapsed < 30.0  # a bounded wait, not a hang
    # the context is still usable: a small symmetric product matches the oracle
    w = inputs.symmetric(3000, 2, seed=9, tie_frac=0.05)
    s, p = L.sort_anchors(dev(w["a"]))
    y = host(L.apply_sym(s, p, dev(w["x"])))
    L.check()
    assert_close(y, oracle.sym_apply(w["a"], w["x"]), oracle.sym_apply(w["a"], w["x"], twin=True), "y after timeout")


def test_check_rejects_a_small_workspace(L):
    import torch
    ws = torch.empty(512, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = L.lib().laplex_check_wait_bound(ws.data_ptr(), ws.numel(), st.data_ptr(), None)
    assert rc == 3  # LAPLEX_ERR_WORKSPACE, before any launch
