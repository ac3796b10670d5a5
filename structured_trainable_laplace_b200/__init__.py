"""LAPLEX exact Laplace-kernel operators on B200 (sm_100a).

The kernels and their C ABI live in liblaplex.so (include/laplex.h); ``laplex``
is the thin torch binding.  ``inputs`` draws the seeded synthetic workloads.
"""
import importlib

from . import inputs  # noqa: F401

__all__ = ["inputs", "laplex"]


def __getattr__(name):
    if name == "laplex":
        return importlib.import_module(__name__ + ".laplex")
    raise AttributeError(name)
