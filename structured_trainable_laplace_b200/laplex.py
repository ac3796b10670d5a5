"""Python binding of liblaplex.so (include/laplex.h): argument marshalling only.

Every function here takes CUDA torch tensors, allocates the outputs and the
scratch workspace with torch (device memory and streams are all torch is used
for), and calls the C ABI entry point of the same name on the current stream.
All arithmetic happens in the library's CUDA kernels.  If the library has not
been built, every call raises: there is no fallback.

Vectors are feature-major [n][B] float32 (a 1-D tensor is B = 1 and comes back
1-D).  Anchors are passed sorted together with their permutation, as returned by
sort_anchors.  Calls do not synchronise; ``check()`` synchronises and raises if
a kernel reported an error (non-finite anchor, bounded wait exceeded).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblaplex.so")

OP_SYM, OP_GENERAL, OP_TRANSPOSE, OP_PHASED, OP_PHASED_TRANSPOSE, OP_GRAM = range(6)
OPS = {"sym": OP_SYM, "general": OP_GENERAL, "transpose": OP_TRANSPOSE, "phased": OP_PHASED,
       "phased_transpose": OP_PHASED_TRANSPOSE, "gram": OP_GRAM}
STATUS = {0: "ok", 1: "invalid argument", 2: "pointer not 16-byte aligned", 3: "workspace too small",
          4: "non-finite anchor", 5: "lookback wait exceeded its bound", 6: "CUDA error"}


class LaplexError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code})")
        self.code = code


_lib = None


def lib():
    """The loaded liblaplex.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m structured_trainable_laplace_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sig = {
            "laplex_status_string": ([I], ctypes.c_char_p),
            "laplex_read_status": ([P, P, P], I),
            "laplex_sort_workspace_size": ([I64], SZ),
            "laplex_sort_anchors": ([P, I64, P, P, P, SZ, P, P], I),
            "laplex_resort_workspace_size": ([I64], SZ),
            "laplex_resort_anchors": ([P, I64, P, P, P, P, SZ, P, P, P], I),
            "laplex_workspace_size": ([I, I64, I64, I64], SZ),
            "laplex_saved_size": ([I, I64, I64, I64], SZ),
            "laplex_apply_sym": ([P, P, I64, P, I64, P, P, P, SZ, P, P], I),
            "laplex_apply_sym_noalloc": ([P, P, I64, P, I64, P, P, P], I),
            "laplex_apply_general": ([P, P, I64, P, P, I64, P, I64, P, P, P, SZ, P, P], I),
            "laplex_apply_transpose": ([P, P, I64, P, P, I64, P, I64, P, P, P, SZ, P, P], I),
            "laplex_apply_phased": ([P, P, I64, P, P, P, I64, P, I, P, I64, P, P, P, SZ, P, P], I),
            "laplex_backward": ([I, P, P, I64, P, P, P, I64, P, P, P, I64, P, P, P, P, P, P, P, SZ, P, P], I),
            "laplex_gram_apply": ([P, P, I64, P, P, I64, P, P, I64, P, P, P, P, P, SZ, P, P], I),
            "laplex_gram_backward": ([P, P, I64, P, P, I64, P, P, P, I64, P, P, P, P, P, SZ, P, P], I),
            "laplex_check_wait_bound": ([P, SZ, P, P], I),
            "laplex_profile_enable": ([I], None),
            "laplex_profile_report": ([I, P, I, P, P], I),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def exported_symbols() -> list:
    """Names of the C entry points this binding calls."""
    return ["laplex_status_string", "laplex_read_status", "laplex_sort_workspace_size", "laplex_sort_anchors",
            "laplex_resort_workspace_size", "laplex_resort_anchors",
            "laplex_workspace_size", "laplex_saved_size", "laplex_apply_sym", "laplex_apply_sym_noalloc",
            "laplex_apply_general",
            "laplex_apply_transpose", "laplex_apply_phased", "laplex_backward", "laplex_gram_apply",
            "laplex_gram_backward", "laplex_check_wait_bound", "laplex_profile_enable", "laplex_profile_report"]


# ---------------------------------------------------------------- plumbing

_ws = {}
_status = {}


def _dev(t: torch.Tensor) -> int:
    return t.device.index if t.device.index is not None else torch.cuda.current_device()


def workspace(nbytes: int, device: int) -> torch.Tensor:
    """A grow-only scratch buffer per (device, current stream): the calls of one
    stream reuse it in stream order, calls on different streams never share it."""
    key = (device, torch.cuda.current_stream(device).cuda_stream)
    buf = _ws.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=f"cuda:{device}")
        _ws[key] = buf
    return buf


def release_workspace(stream=None, device: int | None = None) -> None:
    """Drop the cached scratch of `stream` (default: the current stream), e.g. after
    a side stream or a graph-capture stream is no longer used."""
    device = torch.cuda.current_device() if device is None else device
    stream = torch.cuda.current_stream(device) if stream is None else stream
    _ws.pop((device, stream.cuda_stream), None)


def status_word(device: int) -> torch.Tensor:
    st = _status.get(device)
    if st is None:
        st = torch.zeros(1, dtype=torch.int32, device=f"cuda:{device}")
        _status[device] = st
    return st


def check(device: int | None = None) -> None:
    """Synchronise the current stream and raise if a kernel recorded an error."""
    device = torch.cuda.current_device() if device is None else device
    st = status_word(device)
    h = ctypes.c_int32(0)
    code = lib().laplex_read_status(ctypes.c_void_p(st.data_ptr()), _stream(device), ctypes.byref(h))
    if code != 0:
        st.zero_()
        raise LaplexError(int(code), "kernel status")


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("laplex: tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("laplex: tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device: int):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _rows(x: torch.Tensor):
    if x.dtype != torch.float32:
        raise ValueError("laplex: vectors are float32")
    return (x.reshape(-1, 1), True) if x.dim() == 1 else (x, False)


def _ok(code: int, where: str):
    if code != 0:
        raise LaplexError(int(code), where)


def _out_like_rows(rows: int, B: int, squeeze: bool, device):
    y = torch.empty((rows, B), dtype=torch.float32, device=device)
    return y, (lambda t: t.reshape(-1) if squeeze else t)


# ---------------------------------------------------------------- entry points

def sort_workspace_size(n: int) -> int:
    return int(lib().laplex_sort_workspace_size(n))


def workspace_size(op, n: int, k: int, B: int) -> int:
    return int(lib().laplex_workspace_size(OPS.get(op, op), n, k, B))


def saved_size(op, n: int, k: int, B: int) -> int:
    return int(lib().laplex_saved_size(OPS.get(op, op), n, k, B))


def saved_buffer(op, n: int, k: int, B: int, device) -> torch.Tensor:
    """Caller-owned buffer for a forward to fill and the matching backward to read."""
    return torch.empty(max(saved_size(op, n, k, B), 16), dtype=torch.uint8, device=device)


def sort_anchors(a: torch.Tensor):
    """(a_sorted float32 [n], perm uint32 [n]) with a_sorted[r] = a[perm[r]], stable."""
    n = a.numel()
    d = _dev(a)
    a_sorted = torch.empty(n, dtype=torch.float32, device=a.device)
    perm = torch.empty(n, dtype=torch.uint32, device=a.device)
    nb = sort_workspace_size(n)
    ws = workspace(nb, d)
    _ok(lib().laplex_sort_anchors(_p(a), n, _p(a_sorted), _p(perm), _p(ws), ws.numel(),
                                  _p(status_word(d)), _stream(d)), "sort_anchors")
    return a_sorted, perm


RESORT_PATHS = {0: "sorted", 1: "repaired", 2: "full"}


def resort_workspace_size(n: int) -> int:
    return int(lib().laplex_resort_workspace_size(n))


def resort_anchors(a: torch.Tensor, perm_prev: torch.Tensor, path: torch.Tensor = None):
    """Warm-start re-sort: (a_sorted, perm), identical to sort_anchors(a), from the
    permutation of an earlier sort.  `path` (optional int32 device tensor of one
    element) receives 0 / 1 / 2 = already sorted / repaired / full sort."""
    n = a.numel()
    d = _dev(a)
    if perm_prev.numel() != n:
        raise ValueError("perm_prev must have as many entries as a")
    a_sorted = torch.empty(n, dtype=torch.float32, device=a.device)
    perm = torch.empty(n, dtype=torch.uint32, device=a.device)
    ws = workspace(resort_workspace_size(n), d)
    _ok(lib().laplex_resort_anchors(_p(a), n, _p(perm_prev), _p(a_sorted), _p(perm), _p(ws), ws.numel(),
                                    _p(status_word(d)), _p(path), _stream(d)), "resort_anchors")
    return a_sorted, perm


def apply_sym(a_sorted, perm, x, saved=None):
    """y = K x, K_ij = exp(-|a_i - a_j|)."""
    xr, sq = _rows(x)
    n, B = xr.shape
    d = _dev(x)
    y, back = _out_like_rows(n, B, sq, x.device)
    ws = workspace(workspace_size(OP_SYM, n, 1, B), d)
    _ok(lib().laplex_apply_sym(_p(a_sorted), _p(perm), n, _p(xr), B, _p(y), _p(saved), _p(ws), ws.numel(),
                               _p(status_word(d)), _stream(d)), "apply_sym")
    return back(y)


def apply_sym_noalloc(a_sorted, perm, x):
    """y = K x on the library's static scratch: no workspace (n * padded B <= 2^20)."""
    xr, sq = _rows(x)
    n, B = xr.shape
    d = _dev(x)
    y, back = _out_like_rows(n, B, sq, x.device)
    _ok(lib().laplex_apply_sym_noalloc(_p(a_sorted), _p(perm), n, _p(xr), B, _p(y), _p(status_word(d)), _stream(d)),
        "apply_sym_noalloc")
    return back(y)


def _rect(op, a_sorted, b_sorted, x, out_rows):
    """Rows of x, the output buffer, its reshaping back, and the workspace of a
    rectangular op."""
    xr, sq = _rows(x)
    B = xr.shape[1]
    n, k = a_sorted.numel(), b_sorted.numel()
    d = _dev(x)
    y, back = _out_like_rows(out_rows, B, sq, x.device)
    ws = workspace(workspace_size(op, n, k, B), d)
    return xr, y, back, ws, d, n, k, B


def apply_general(a_sorted, perm_a, b_sorted, perm_b, x, saved=None):
    """y = E x with E_ij = exp(-|a_i - b_j|); x [k][B] -> y [n][B]."""
    xr, y, back, ws, d, n, k, B = _rect(OP_GENERAL, a_sorted, b_sorted, x, a_sorted.numel())
    _ok(lib().laplex_apply_general(_p(a_sorted), _p(perm_a), n, _p(b_sorted), _p(perm_b), k, _p(xr), B, _p(y),
                                   _p(saved), _p(ws), ws.numel(), _p(status_word(d)), _stream(d)), "apply_general")
    return back(y)


def apply_transpose(a_sorted, perm_a, b_sorted, perm_b, x, saved=None):
    """z = E^T x; x [n][B] -> z [k][B]."""
    xr, z, back, ws, d, n, k, B = _rect(OP_TRANSPOSE, a_sorted, b_sorted, x, b_sorted.numel())
    _ok(lib().laplex_apply_transpose(_p(a_sorted), _p(perm_a), n, _p(b_sorted), _p(perm_b), k, _p(xr), B, _p(z),
                                     _p(saved), _p(ws), ws.numel(), _p(status_word(d)), _stream(d)),
        "apply_transpose")
    return back(z)


def apply_phased(a_sorted, perm_a, phi, b_sorted, perm_b, psi, x, transpose=False, saved=None):
    """Phased operator E_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j); transpose selects E^T."""
    op = OP_PHASED_TRANSPOSE if transpose else OP_PHASED
    rows = b_sorted.numel() if transpose else a_sorted.numel()
    xr, out, back, ws, d, n, k, B = _rect(op, a_sorted, b_sorted, x, rows)
    _ok(lib().laplex_apply_phased(_p(a_sorted), _p(perm_a), n, _p(phi), _p(b_sorted), _p(perm_b), k, _p(psi),
                                  int(bool(transpose)), _p(xr), B, _p(out), _p(saved), _p(ws), ws.numel(),
                                  _p(status_word(d)), _stream(d)), "apply_phased")
    return back(out)


def backward(op, a_sorted, perm_a, x, g, b_sorted=None, perm_b=None, phi=None, psi=None, saved=None,
             need=("gx", "ga", "gb", "gphi", "gpsi")):
    """Gradients of <g, out> for the forward `op` (name or number).  Returns a dict
    with the requested entries among gx, ga, gb, gphi, gpsi."""
    op = OPS.get(op, op)
    xr, sq = _rows(x)
    gr, _ = _rows(g)
    B = xr.shape[1]
    n = a_sorted.numel()
    k = b_sorted.numel() if b_sorted is not None else 1
    d = _dev(x)
    dev = x.device
    phased = op in (OP_PHASED, OP_PHASED_TRANSPOSE)
    rect = op != OP_SYM
    out = {}
    if "gx" in need:
        out["gx"] = torch.empty_like(xr)
    if "ga" in need:
        out["ga"] = torch.empty(n, dtype=torch.float32, device=dev)
    if rect and "gb" in need:
        out["gb"] = torch.empty(k, dtype=torch.float32, device=dev)
    if phased and "gphi" in need:
        out["gphi"] = torch.empty(n, dtype=torch.float32, device=dev)
    if phased and "gpsi" in need:
        out["gpsi"] = torch.empty(k, dtype=torch.float32, device=dev)
    ws = workspace(workspace_size(op, n, k, B), d)
    _ok(lib().laplex_backward(op, _p(a_sorted), _p(perm_a), n, _p(phi), _p(b_sorted), _p(perm_b), k, _p(psi),
                              _p(xr), _p(gr), B, _p(saved), _p(out.get("gx")), _p(out.get("ga")), _p(out.get("gb")),
                              _p(out.get("gphi")), _p(out.get("gpsi")), _p(ws), ws.numel(), _p(status_word(d)),
                              _stream(d)), "backward")
    if "gx" in out and sq:
        out["gx"] = out["gx"].reshape(-1)
    return out


def gram_apply(a_sorted, perm_a, b_sorted, perm_b, D, v, g=None, return_w=False):
    """y = A diag(D) A^T v (A_ij = exp(-|a_i - b_j|)); with g also gD.  Returns y,
    or a tuple (y, w) / (y, gD) / (y, w, gD) following return_w and g."""
    vr, sq = _rows(v)
    n, B = vr.shape
    k = b_sorted.numel()
    d = _dev(v)
    y = torch.empty_like(vr)
    w = torch.empty((k, B), dtype=torch.float32, device=v.device) if return_w else None
    gr = _rows(g)[0] if g is not None else None
    gD = torch.empty(k, dtype=torch.float32, device=v.device) if g is not None else None
    ws = workspace(workspace_size(OP_GRAM, n, k, B), d)
    _ok(lib().laplex_gram_apply(_p(a_sorted), _p(perm_a), n, _p(b_sorted), _p(perm_b), k, _p(D), _p(vr), B, _p(y),
                                _p(w), _p(gr), _p(gD), _p(ws), ws.numel(), _p(status_word(d)), _stream(d)),
        "gram_apply")
    y = y.reshape(-1) if sq else y
    res = (y,)
    if return_w:
        res += (w,)
    if g is not None:
        res += (gD,)
    return res[0] if len(res) == 1 else res


def gram_backward(a_sorted, perm_a, b_sorted, perm_b, D, v, g, need=("gv", "ga", "gb", "gD")):
    """Gradients of <g, A diag(D) A^T v>: a dict with the requested entries among
    gv [n][B], ga [n], gb [k], gD [k]."""
    vr, sq = _rows(v)
    gr, _ = _rows(g)
    n, B = vr.shape
    k = b_sorted.numel()
    d = _dev(v)
    dev = v.device
    out = {}
    if "gv" in need:
        out["gv"] = torch.empty_like(vr)
    if "ga" in need:
        out["ga"] = torch.empty(n, dtype=torch.float32, device=dev)
    if "gb" in need:
        out["gb"] = torch.empty(k, dtype=torch.float32, device=dev)
    if "gD" in need:
        out["gD"] = torch.empty(k, dtype=torch.float32, device=dev)
    ws = workspace(workspace_size(OP_GRAM, n, k, B), d)
    _ok(lib().laplex_gram_backward(_p(a_sorted), _p(perm_a), n, _p(b_sorted), _p(perm_b), k, _p(D), _p(vr), _p(gr), B,
                                   _p(out.get("gv")), _p(out.get("ga")), _p(out.get("gb")), _p(out.get("gD")), _p(ws),
                                   ws.numel(), _p(status_word(d)), _stream(d)), "gram_backward")
    if "gv" in out and sq:
        out["gv"] = out["gv"].reshape(-1)
    return out


# ---------------------------------------------------------------- diagnostics

def check_wait_bound(device: int | None = None) -> int:
    """Run the failure-detection self-check (a bounded lookback wait on a flag that
    nothing sets) on its own status word and return the status it recorded (5 =
    the wait gave up, as it must)."""
    device = torch.cuda.current_device() if device is None else device
    ws = torch.empty(1024, dtype=torch.uint8, device=f"cuda:{device}")
    st = torch.zeros(1, dtype=torch.int32, device=f"cuda:{device}")
    _ok(lib().laplex_check_wait_bound(_p(ws), ws.numel(), _p(st), _stream(device)), "check_wait_bound")
    h = ctypes.c_int32(0)
    lib().laplex_read_status(ctypes.c_void_p(st.data_ptr()), _stream(device), ctypes.byref(h))
    return int(h.value)


# ---------------------------------------------------------------- tracing

def profile_enable(on: bool = True) -> None:
    """Start (clearing the record) or stop bracketing every kernel launch with CUDA events."""
    lib().laplex_profile_enable(int(bool(on)))


def profile_report(max_kernels: int = 64) -> dict:
    """{kernel name: (launches, total device ms)} since profile_enable(True); clears the record."""
    names = ctypes.create_string_buffer(max_kernels * 32)
    launches = (ctypes.c_int * max_kernels)()
    ms = (ctypes.c_double * max_kernels)()
    nk = lib().laplex_profile_report(max_kernels, names, 32, launches, ms)
    if nk < 0:
        raise LaplexError(6, "profile_report")
    out = {}
    for i in range(min(nk, max_kernels)):
        name = names.raw[i * 32:(i + 1) * 32].split(b"\0", 1)[0].decode()
        out[name] = (int(launches[i]), float(ms[i]))
    return out
