"""Comparison metrics used by the parity tests.

max-abs relative error = max |got - ref| / max |ref| over a tensor; cosine
similarity over the flattened tensor."""

import numpy as np


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (den if den > 0 else 1.0))


def cosine(got, ref) -> float:
    a = np.asarray(got, dtype=np.float64).ravel()
    b = np.asarray(ref, dtype=np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))


# Tolerances: fp32 path 1e-4, bf16 path 2e-2 with cosine >= 0.999.
TOL_F32 = 1e-4
TOL_BF16 = 2e-2
COS_BF16 = 0.999


def noise_floor(name: str) -> dict:
    """The oracle's own bf16 noise floor for a model (tests/golden/noise_floor.json)."""
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "noise_floor.json")
    with open(path) as f:
        return json.load(f)[name]
