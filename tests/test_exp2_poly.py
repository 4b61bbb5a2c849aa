"""The cubic 2^f that the flash-attention softmax evaluates on the FMA pipe:
its fp32 constants in attn_tc.cu are the minimax fit that exp2_poly_fit.py
computes, and the kernel's evaluation (nearest-integer split with the
1.5 * 2^23 shift, cubic, exponent added to the bits), emulated here in fp32,
stays within the fit's error over the whole input range the softmax feeds it."""

import importlib.util
import pathlib
import re

import numpy as np

CSRC = pathlib.Path(__file__).resolve().parents[1] / "looped_weight_shared_b200" / "csrc"


def _kernel_constants():
    src = (CSRC / "attn_tc.cu").read_text()
    vals = {}
    for k in range(4):
        m = re.search(rf"P2_C{k} = ([0-9.eE+-]+)f", src)
        assert m, f"P2_C{k} not found"
        vals[k] = np.float32(float(m.group(1)))
    return [vals[k] for k in range(4)]


def _fit():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", CSRC / "exp2_poly_fit.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.fit()


def _kernel_exp2(x: np.ndarray, c) -> np.ndarray:
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (np.float64(p) * f + c[k]).astype(np.float32)  # one rounding, like an FMA
    bits = (p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_constants_are_the_fit():
    c_fit, err = _fit()
    assert err < 7.5e-5
    assert [float(v) for v in _kernel_constants()] == [float(v) for v in c_fit]


def test_evaluation_error_over_softmax_range():
    c = _kernel_constants()
    x = np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32)
    got = _kernel_exp2(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 7.5e-5
    # integers are exact up to the cubic's value at f = 0
    xi = np.arange(-125, 9, dtype=np.float32)
    assert np.all(np.abs(_kernel_exp2(xi, c) / np.exp2(xi.astype(np.float64)) - 1.0) < 7.5e-5)
    # below the clamp the result is 2^-125 (tiny, never 0 or garbage)
    low = _kernel_exp2(np.array([-126.0, -1e4, -np.inf], dtype=np.float32), c)
    assert np.all((low > 0) & (low < 3e-38))
