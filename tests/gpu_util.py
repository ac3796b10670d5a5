"""GPU-side plumbing for the parity tests: run the CUDA path through the binding."""
from __future__ import annotations

import numpy as np
import pytest


def laplex_or_fail():
    """The binding with the library built; on a GPU machine a missing library fails the test."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from structured_trainable_laplace_b200 import build, laplex
    build.build()
    laplex.lib()
    return laplex


def dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    import torch
    if t.dtype == torch.uint32:
        return t.view(torch.int32).cpu().numpy().view(np.uint32)
    return t.cpu().numpy()
