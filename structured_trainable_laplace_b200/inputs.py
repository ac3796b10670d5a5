"""Seeded synthetic inputs for the LAPLEX operators.

This module draws random anchors, phases, weights and vectors with the shapes and
distributions of the workloads described for LAPLEX ("LAPLEX: The FFT of Learnable
Laplace Kernels", gist.science technical summary, sections 4.1-4.3: a symmetric
operator at scale, a phased classification head, a Gram/covariance operator on a
flattened image).  It holds none of the operators' arithmetic: it only produces
numbers.  Both the fp64 oracle (through the tests) and the CUDA path consume its
output, so the two sides always see identical inputs.

Recipe (all draws from ``numpy.random.Generator`` streams spawned from one
``SeedSequence(seed)`` in the fixed order a, x, g, b, phi, psi, d, ties):

* uniform anchors are drawn in fp64 and cast to fp32;
* normal vectors use ``standard_normal(dtype=float32)``;
* vectors are feature-major ``[n][B]`` float32 (row i holds the B batch values of
  feature i);
* the tie recipe overwrites ``round(frac * n)`` distinct targets, each with a copy
  of the original value at a source index drawn uniformly from the non-targets.

Large arrays are drawn in chunks into preallocated buffers, so host memory stays
at the size of the result.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

_STREAMS = ("a", "x", "g", "b", "phi", "psi", "d", "ties")
_CHUNK = 1 << 24


def streams(seed: int) -> dict:
    """One independent generator per input, spawned in a fixed order."""
    kids = np.random.SeedSequence(seed).spawn(len(_STREAMS))
    return {name: np.random.default_rng(k) for name, k in zip(_STREAMS, kids)}


def uniform(rng: np.random.Generator, n: int, lo: float, hi: float) -> np.ndarray:
    """fp32 array of n draws from U[lo, hi), drawn in fp64 then cast."""
    out = np.empty(n, dtype=np.float32)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = rng.uniform(lo, hi, size=e - s)
    return out


def normal(rng: np.random.Generator, shape) -> np.ndarray:
    """fp32 standard normals of the given shape (row-major), drawn in chunks."""
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape(-1)
    for s in range(0, flat.size, _CHUNK):
        e = min(flat.size, s + _CHUNK)
        flat[s:e] = rng.standard_normal(e - s, dtype=np.float32)
    return out


def overwrite_with_copies(rng: np.random.Generator, a: np.ndarray, frac: float) -> np.ndarray:
    """Make ties: round(frac*n) distinct targets take the value of a non-target source."""
    n = a.shape[0]
    m = int(round(frac * n))
    if m == 0 or m >= n:
        return a
    targets = rng.choice(n, size=m, replace=False)
    mask = np.ones(n, dtype=bool)
    mask[targets] = False
    pool = np.nonzero(mask)[0]
    sources = pool[rng.integers(0, pool.size, size=m)]
    out = a.copy()
    out[targets] = a[sources]
    return out


def softplus(z: np.ndarray) -> np.ndarray:
    """Positive weights for the Gram operator's diagonal D (a data-generation step)."""
    z64 = z.astype(np.float64)
    return (np.maximum(z64, 0.0) + np.log1p(np.exp(-np.abs(z64)))).astype(np.float32)


@dataclass
class Workload:
    """A named set of inputs.  Keys follow the operators' notation."""

    name: str
    op: str
    n: int
    B: int
    k: int = 0
    arrays: dict = field(default_factory=dict)

    def __getitem__(self, key):
        return self.arrays[key]

    def __contains__(self, key):
        return key in self.arrays


def moved(a: np.ndarray, step: float, seed: int = 1) -> np.ndarray:
    """The anchors after one training update: a + step * N(0, 1), rounded to fp32
    (a stand-in for a gradient step on trainable anchors)."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x6d6f7665]))
    out = np.empty_like(a, dtype=np.float32)
    for s in range(0, a.size, _CHUNK):
        e = min(a.size, s + _CHUNK)
        out[s:e] = (a[s:e].astype(np.float64) + step * rng.standard_normal(e - s)).astype(np.float32)
    return out


def symmetric(n: int, B: int, seed: int = 0, spacing: float = 0.05, tie_frac: float = 0.0,
              with_g: bool = True, name: str = "symmetric") -> Workload:
    """a ~ U[0, spacing*n], x, g ~ N(0,1) [n][B]; optional copies to make ties."""
    r = streams(seed)
    a = uniform(r["a"], n, 0.0, spacing * n)
    if tie_frac > 0:
        a = overwrite_with_copies(r["ties"], a, tie_frac)
    arrays = {"a": a, "x": normal(r["x"], (n, B))}
    if with_g:
        arrays["g"] = normal(r["g"], (n, B))
    return Workload(name, "sym", n, B, 0, arrays)


def phased_head(n: int, k: int, B: int, seed: int = 0, span: float = 100.0,
                name: str = "phased_head") -> Workload:
    """Rectangular phased head: a, b ~ U[0, span], phi, psi ~ U[0, 2pi), x [n][B], h [k][B]."""
    r = streams(seed)
    arrays = {
        "a": uniform(r["a"], n, 0.0, span),
        "x": normal(r["x"], (n, B)),
        "h": normal(r["g"], (k, B)),
        "b": uniform(r["b"], k, 0.0, span),
        "phi": uniform(r["phi"], n, 0.0, 2.0 * math.pi),
        "psi": uniform(r["psi"], k, 0.0, 2.0 * math.pi),
    }
    return Workload(name, "phased_transpose", n, B, k, arrays)


def gram(n: int, k: int, B: int, seed: int = 0, span: float = 1000.0, name: str = "gram") -> Workload:
    """Gram/covariance apply: a, b ~ U[0, span], D = softplus(N(0,1)), v, g ~ N(0,1) [n][B]."""
    r = streams(seed)
    arrays = {
        "a": uniform(r["a"], n, 0.0, span),
        "v": normal(r["x"], (n, B)),
        "g": normal(r["g"], (n, B)),
        "b": uniform(r["b"], k, 0.0, span),
        "D": softplus(normal(r["d"], (k,))),
    }
    return Workload(name, "gram", n, B, k, arrays)


def rectangular(n: int, k: int, B: int, seed: int = 0, span_a: float = 100.0, span_b: float = 100.0,
                phased: bool = False, transpose: bool = False, name: str = "rectangular") -> Workload:
    """General rectangular operator inputs.  Inputs sit at b (k rows) unless transpose,
    where they sit at a (n rows); the upstream gradient g sits on the output side."""
    r = streams(seed)
    rows_in, rows_out = (n, k) if transpose else (k, n)
    arrays = {
        "a": uniform(r["a"], n, 0.0, span_a),
        "x": normal(r["x"], (rows_in, B)),
        "g": normal(r["g"], (rows_out, B)),
        "b": uniform(r["b"], k, 0.0, span_b),
    }
    if phased:
        arrays["phi"] = uniform(r["phi"], n, 0.0, 2.0 * math.pi)
        arrays["psi"] = uniform(r["psi"], k, 0.0, 2.0 * math.pi)
    op = ("phased_" if phased else "general_") + ("transpose" if transpose else "forward")
    return Workload(name, op, n, B, k, arrays)


def device_symmetric(n: int, B: int, device, seed: int = 0, spacing: float = 0.05, name: str = "symmetric"):
    """The symmetric recipe (a ~ U[0, spacing*n], x, g ~ N(0,1) [n][B]) drawn
    directly on a CUDA device with torch's seeded generator, for sizes whose host
    draw and upload would take longer than the measurement (n = 10^9).  Same
    distributions as ``symmetric`` (not the same numbers).  Returns (Workload
    without host arrays, dict of device tensors a, x, g)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    a = torch.empty(n, dtype=torch.float32, device=device)
    a.uniform_(0.0, spacing * n, generator=gen)
    x = torch.empty((n, B), dtype=torch.float32, device=device)
    x.normal_(generator=gen)
    g = torch.empty((n, B), dtype=torch.float32, device=device)
    g.normal_(generator=gen)
    return Workload(name, "sym", n, B, 0, {}), {"a": a, "x": x, "g": g}


# The five named workloads.  Sizes and distributions are the ones stated for each.
def sym_small_ties(seed: int = 0) -> Workload:
    """n=4096, a ~ U[0, 0.05n] with 5% overwritten by copies of other anchors, B=1."""
    return symmetric(4096, 1, seed, tie_frac=0.05, name="sym_n4096_b1_ties5pct")


def sym_2p24_b16(seed: int = 0, n: int = 1 << 24) -> Workload:
    """n=2^24, a ~ U[0, 0.05n], B=16 (symmetric forward+backward)."""
    return symmetric(n, 16, seed, name=f"sym_n{n}_b16")


def phased_head_2p22(seed: int = 0, n: int = 1 << 22, k: int = 1024, B: int = 128) -> Workload:
    """n=2^22 -> k=1024 phased head, anchors U[0,100], phases U[0,2pi), B=128."""
    return phased_head(n, k, B, seed, name=f"phased_head_n{n}_k{k}_b{B}")


def gram_image(seed: int = 0, n: int = 3 * 1024 * 1024, k: int = 65536, B: int = 8) -> Workload:
    """Gram apply on a flattened 3x1024x1024 image: n=3,145,728, k=65,536, B=8."""
    return gram(n, k, B, seed, name=f"gram_n{n}_k{k}_b{B}")


def sym_extreme(seed: int = 0, n: int = 10 ** 9) -> Workload:
    """n=10^9 symmetric, B=1, a ~ U[0, 0.05n]."""
    return symmetric(n, 1, seed, name=f"sym_n{n}_b1")
