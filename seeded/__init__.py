"""Seeded synthetic inputs shared by the tests, the oracle runs and the bench.

This module only draws numbers; it holds none of the looped decoder's
arithmetic.  The generator is SplitMix64 (Steele, Lea and Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014; finaliser constants
as published with Vigna's reference implementation) used as a counter-based
stream:

    key(seed, stream) = mix64(mix64(seed) + stream)          (mod 2**64)
    u64(seed, stream, j) = mix64(key + (j + 1) * 0x9E3779B97F4A7C15)

so any element of any tensor can be drawn without drawing the others.

Derived draws (each side of the parity tests implements these same rules on
its own; only this module is shared):

* uniform double  u(j)  = (u64(j) >> 11) * 2**-53                 in [0, 1)
* normal element i      : Box-Muller on the pair p = i // 2 with
                          u1 = ((u64(2p) >> 11) + 1) * 2**-53     in (0, 1]
                          u2 = (u64(2p + 1) >> 11) * 2**-53
                          r = sqrt(-2 ln u1), t = 2 pi u2,
                          z = r cos t (i even) or r sin t (i odd), in fp64
* a weight               = 0.02 * z, fp64 -> fp32 (nearest) [-> bf16 (nearest even)]
* a token                = ((u64(j) >> 32) * vocab) >> 32        (multiply-high)

Stream ids name tensors: see ``stream_id``.  Matrices are stored [out, in]
(row = output feature) and element (o, i) is counter index o * in + i.
"""

from __future__ import annotations

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1

# Tensor kinds inside one physical layer (stream = 1000 + 100 * layer + kind).
K_WQ, K_WK, K_WV, K_WG, K_WO, K_WGATE, K_WUP, K_WDOWN = 1, 2, 3, 4, 5, 7, 8, 9
S_EMBED = 1
S_TOKENS = 7
S_HIDDEN = 8
S_DECODE_TOKENS = 9


def layer_stream(layer: int, kind: int) -> int:
    return 1000 + 100 * layer + kind


def site_stream(site: int) -> int:
    """Stream of the mHC projection Phi of coefficient site ``site``.

    Site = 2 * (physical layer - n_prelude) + sublayer (0 attention, 1 FFN)."""
    return 100000 + 10 * site + 1


def _mix64_int(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= np.uint64(0xBF58476D1CE4E5B9)
        z ^= z >> np.uint64(27)
        z *= np.uint64(0x94D049BB133111EB)
        z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, stream: int) -> int:
    return _mix64_int((_mix64_int(seed) + stream) & _M64)


def u64(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    key = np.uint64(stream_key(seed, stream))
    j = np.arange(start, start + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        s = key + (j + np.uint64(1)) * np.uint64(GAMMA)
    return _mix64(s)


def splitmix64_sequence(state: int, n: int) -> list[int]:
    """The plain SplitMix64 sequence from a 64-bit state (for published vectors)."""
    out = []
    for _ in range(n):
        state = (state + GAMMA) & _M64
        out.append(_mix64_int(state))
    return out


def uniform(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    return (u64(seed, stream, start, n) >> np.uint64(11)).astype(np.float64) * 2.0**-53


def normal(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    """Standard normals for elements [start, start + n) of a stream (fp64)."""
    if n == 0:
        return np.zeros(0)
    p0 = start // 2
    p1 = (start + n - 1) // 2 + 1
    raw = u64(seed, stream, 2 * p0, 2 * (p1 - p0))
    u1 = ((raw[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0**-53
    u2 = (raw[1::2] >> np.uint64(11)).astype(np.float64) * 2.0**-53
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    z = np.empty(2 * (p1 - p0))
    z[0::2] = r * np.cos(t)
    z[1::2] = r * np.sin(t)
    off = start - 2 * p0
    return z[off:off + n]


def to_bf16_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even), returned as fp32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    b = (b + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return b.astype(np.uint32).view(np.float32)


def weights(seed: int, stream: int, n: int, bf16: bool, scale: float = 0.02) -> np.ndarray:
    """A weight tensor: 0.02 * normal, fp64 -> fp32 (-> bf16), as fp32 values."""
    w = (scale * normal(seed, stream, 0, n)).astype(np.float32)
    return to_bf16_f32(w) if bf16 else w


def tokens(seed: int, batch: int, seq: int, vocab: int, stream: int = S_TOKENS) -> np.ndarray:
    raw = u64(seed, stream, 0, batch * seq)
    t = ((raw >> np.uint64(32)) * np.uint64(vocab)) >> np.uint64(32)
    return t.astype(np.int32).reshape(batch, seq)


def hidden(seed: int, batch: int, seq: int, dim: int) -> np.ndarray:
    """Hidden-state inputs h ~ N(0, 1), fp32, [batch, seq, dim]."""
    return normal(seed, S_HIDDEN, 0, batch * seq * dim).astype(np.float32).reshape(batch, seq, dim)
