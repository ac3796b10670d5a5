"""Reader for the hand-derived worked examples in worked_examples.txt."""
from __future__ import annotations

import math
import os

import numpy as np

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "worked_examples.txt")
_NS = {"e": math.e, "exp": math.exp, "cos": math.cos, "sin": math.sin, "pi": math.pi, "__builtins__": {}}
_INPUTS = {"a", "b", "x", "g", "phi", "psi", "D", "v"}


def load(path: str = _PATH) -> dict:
    """Sections of name -> {key: array}.  Input lines are numbers, expected lines expressions."""
    out, cur = {}, None
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("[") and line.endswith("]"):
                cur = out.setdefault(line[1:-1], {})
                continue
            key, val = (t.strip() for t in line.split("=", 1))
            if key in _INPUTS:
                cur[key] = np.array([float(t) for t in val.split()], dtype=np.float32)
            else:
                cur[key] = np.array([eval(t, _NS) for t in val.split(";")], dtype=np.float64)
    return out
