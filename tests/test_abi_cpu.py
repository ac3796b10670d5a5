"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/laplex.h declares, answers size queries, and rejects bad
arguments before launching anything."""
import ctypes
import os
import re

import pytest

from structured_trainable_laplace_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "laplex.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(laplex_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from structured_trainable_laplace_b200 import laplex
    build_mod.build()
    return laplex.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("laplex_sort_anchors", "laplex_apply_sym", "laplex_apply_general", "laplex_apply_phased",
                     "laplex_apply_transpose", "laplex_backward", "laplex_gram_apply"):
        assert required in names


def test_library_exports_every_declared_function(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_binding_covers_the_header():
    from structured_trainable_laplace_b200 import laplex
    assert set(laplex.exported_symbols()) == set(declared_functions())


def test_status_strings(L):
    assert L.laplex_status_string(0) == b"ok"
    assert L.laplex_status_string(5) == b"lookback wait exceeded its bound"


def test_size_queries(L):
    from structured_trainable_laplace_b200 import laplex
    assert laplex.sort_workspace_size(1 << 24) >= 8 * (1 << 24)
    # the re-sort's workspace also holds the full sort's (its fallback)
    assert laplex.resort_workspace_size(1 << 24) >= laplex.sort_workspace_size(1 << 24)
    assert laplex.resort_workspace_size(0) == 0
    assert laplex.workspace_size("sym", 1 << 24, 1, 16) > 0
    assert laplex.saved_size("sym", 1 << 24, 1, 16) > 0
    assert laplex.workspace_size("phased_transpose", 1 << 22, 1024, 128) > 0
    assert laplex.workspace_size("gram", 3 << 20, 65536, 8) > 0
    assert laplex.workspace_size("sym", 0, 1, 1) == 0       # n out of range
    assert laplex.workspace_size("sym", 10, 1, 1025) == 0   # B out of range
    assert laplex.workspace_size(99, 10, 10, 1) == 0        # unknown op


def test_bad_arguments_are_rejected_before_launch(L):
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: the checks fail first
    ws = P(1 << 21)
    # n = 0
    assert L.laplex_apply_sym(fake, fake, 0, fake, 1, ws, None, ws, 1 << 30, None, None) == 1
    # NULL x
    assert L.laplex_apply_sym(fake, fake, 8, None, 1, ws, None, ws, 1 << 30, None, None) == 1
    # workspace too small
    assert L.laplex_apply_sym(fake, fake, 8, fake, 1, ws, None, ws, 8, None, None) == 3
    # misaligned output
    assert L.laplex_apply_sym(P(1 << 20), P(1 << 22), 8, P(1 << 23), 1, P((1 << 24) + 4), None, P(1 << 25),
                              1 << 30, None, None) == 2
    # output overlapping the input
    assert L.laplex_apply_sym(P(1 << 20), P(1 << 22), 8, P(1 << 23), 1, P(1 << 23), None, P(1 << 25), 1 << 30,
                              None, None) == 1
    # phased without phases
    assert L.laplex_apply_phased(fake, fake, 8, None, fake, fake, 4, None, 0, fake, 1, ws, None, ws, 1 << 30,
                                 None, None) == 1
    # gram: g without gD
    assert L.laplex_gram_apply(fake, fake, 8, fake, fake, 4, fake, fake, 1, ws, None, fake, None, ws, 1 << 30,
                               None, None) == 1
    # backward of an unknown op
    assert L.laplex_backward(42, fake, fake, 8, None, fake, fake, 4, None, fake, fake, 1, None, ws, None, None,
                             None, None, ws, 1 << 30, None, None) == 1
    # static-scratch product: beyond its size limit (n * padded B > 2^20)
    assert L.laplex_apply_sym_noalloc(fake, fake, 65537, fake, 16, P(1 << 24), None, None) == 3
    assert L.laplex_apply_sym_noalloc(fake, fake, 4097, fake, 257, P(1 << 24), None, None) == 3
    # sort: n too large
    assert L.laplex_sort_anchors(fake, 1 << 33, fake, fake, ws, 1 << 30, None, None) == 1
    # warm-start re-sort: NULL previous permutation, small workspace, misaligned
    # output, output overlapping perm_prev
    big = 1 << 30
    assert L.laplex_resort_anchors(fake, 8, None, fake, fake, ws, big, None, None, None) == 1
    assert L.laplex_resort_anchors(P(1 << 20), 8, P(1 << 22), P(1 << 23), P(1 << 24), P(1 << 25), 64, None, None,
                                   None) == 3
    assert L.laplex_resort_anchors(P(1 << 20), 8, P(1 << 22), P((1 << 23) + 4), P(1 << 24), P(1 << 25), big, None,
                                   None, None) == 2
    assert L.laplex_resort_anchors(P(1 << 20), 8, P(1 << 22), P(1 << 22), P(1 << 24), P(1 << 25), big, None, None,
                                   None) == 1
