"""laplex_apply_sym_noalloc (the symmetric product on the library's static scratch)
against laplex_apply_sym, through the C ABI: two calls in a row must each agree
with the workspace entry point and with the fp64 oracle, at sizes up to the
entry point's limit (n * padded B = 2^20).  This file is collected last so that
the static scratch is exercised after every other test has used the library."""
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


CASES = [
    ("ties n4096 B1", lambda: inputs.sym_small_ties(0)),
    ("n65499 B16 ragged", lambda: inputs.sym_2p24_b16(5, n=65499)),
    ("n65536 B16 at the limit", lambda: inputs.sym_2p24_b16(6, n=65536)),
    ("n8000 B100", lambda: inputs.symmetric(8000, 100, 7)),  # padded B = 128
]


@pytest.mark.parametrize("tag,make", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_entry(L, tag, make):
    w = make()
    a, x = w["a"], w["x"]
    s, p = L.sort_anchors(dev(a))
    xd = dev(x)
    y_ws = host(L.apply_sym(s, p, xd))
    ref, twin = oracle.sym_apply(a, x), oracle.sym_apply(a, x, twin=True)
    for call in range(2):
        y = host(L.apply_sym_noalloc(s, p, xd))
        L.check()
        assert_close(y, y_ws.reshape(y.shape), twin, f"{tag}: call {call} vs laplex_apply_sym")
        assert_close(y, ref, twin, f"{tag}: call {call} vs oracle")


def test_noalloc_rejects_sizes_beyond_its_scratch(L):
    import torch
    n, B = 65537, 16  # n * 16 = 2^20 + 16
    a = torch.zeros(n, device="cuda")
    p = torch.zeros(n, dtype=torch.int32, device="cuda")
    x = torch.zeros(n, B, device="cuda")
    y = torch.empty_like(x)
    rc = L.lib().laplex_apply_sym_noalloc(a.data_ptr(), p.data_ptr(), n, x.data_ptr(), B, y.data_ptr(), None, None)
    assert rc == 3  # LAPLEX_ERR_WORKSPACE, returned before any launch
