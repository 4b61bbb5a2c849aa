"""ctypes binding of the CPU oracle: TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may
import this package.  It compiles ``oracle.cpp`` with g++ on first use (or in
``__graft_entry__.build()``) and shares no code with the CUDA library.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_DIR, "oracle.cpp")
_HDR = os.path.join(_DIR, "oracle.h")
_LIB = os.path.join(_DIR, "_oracle.so")
_lock = threading.Lock()
_lib = None

FULL, LINEAR = 1, 0
PRELUDE, BLOCK, CODA = 0, 1, 2
ALL_POSITIONS = 1


class Config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "n_prelude", "n_block", "n_loops", "n_coda", "group", "full_slot", "hidden", "ffn", "vocab",
        "n_q", "n_kv", "head_dim", "n_lin", "lin_dim", "lin_chunk", "n_streams", "sinkhorn_iters")] + [
        ("rope_base", C.c_float), ("norm_eps", C.c_float)] + [
        (n, C.c_int32) for n in ("dtype", "io_mode", "max_batch", "max_ctx", "kv_pages")]


def make_config(**kw) -> Config:
    c = Config()
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/_oracle.so (plain g++, OpenMP, no fast-math)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= newest:
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-o", tmp, _SRC]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(_LIB)
            P = C.POINTER
            d, f, i32, i64, u32, u64 = C.c_double, C.c_float, C.c_int32, C.c_int64, C.c_uint32, C.c_uint64
            vp = C.c_void_p
            sig = {
                "oracle_rng_u64": (u64, [u64, u64, u64]),
                "oracle_rng_normal": (d, [u64, u64, u64]),
                "oracle_exp_spec": (f, [f]),
                "oracle_sinkhorn_f32": (None, [vp, vp, i64, i32, i32]),
                "oracle_sinkhorn_f64": (None, [vp, vp, i64, i32, i32]),
                "oracle_num_exec": (i32, [P(Config)]),
                "oracle_schedule": (i32, [P(Config), vp]),
                "oracle_rmsnorm": (None, [vp, vp, vp, i64, i32, d]),
                "oracle_gla_recurrent": (None, [vp, vp, vp, vp, vp, vp, i32, i32, i32]),
                "oracle_attention_naive": (None, [vp, vp, vp, vp, i32, i32, i32, i32]),
                "oracle_rope": (None, [vp, i32, i32, i32, vp, d]),
                "oracle_mhc_site": (None, [vp, vp, vp, vp, i32, i32, i32, d, vp, vp]),
                "oracle_mhc_write": (None, [vp, vp, vp, i32, i32]),
                "oracle_model_create": (vp, [P(Config), u64, vp]),
                "oracle_num_weights": (i32, [P(Config)]),
                "oracle_weight_numel": (i64, [vp, i32]),
                "oracle_get_weight": (i32, [vp, i32, vp]),
                "oracle_prefill": (i32, [vp, vp, vp, i32, i32, vp, u32]),
                "oracle_decode_step": (i32, [vp, vp, i32, vp]),
                "oracle_seq_len": (i32, [vp, i32]),
                "oracle_cache_read": (i32, [vp, i32, i32, i32, i32, vp]),
                "oracle_model_destroy": (None, [vp]),
                "oracle_attention_sublayer": (i32, [P(Config), vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp]),
                "oracle_gla_sublayer": (i32, [P(Config), vp, vp, vp, vp, vp, vp, vp, i32, i32, vp]),
                "oracle_ffn_sublayer": (i32, [P(Config), vp, vp, vp, vp, i64, vp]),
                "oracle_cache_write": (i32, [vp, i32, i32, i32, i32, vp]),
                "oracle_set_seq_len": (i32, [vp, i32, i32]),
                "oracle_set_weight": (i32, [vp, i32, vp]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def rng_u64(seed: int, stream: int, j: int) -> int:
    return lib().oracle_rng_u64(seed, stream, j)


def rng_normal(seed: int, stream: int, i: int) -> float:
    return lib().oracle_rng_normal(seed, stream, i)


def exp_spec(x: float) -> float:
    return lib().oracle_exp_spec(x)


def sinkhorn_f32(logits: np.ndarray, iters: int = 20) -> np.ndarray:
    x = np.ascontiguousarray(logits, dtype=np.float32)
    n = x.shape[-1]
    out = np.empty_like(x)
    lib().oracle_sinkhorn_f32(_p(x), _p(out), x.size // (n * n), n, iters)
    return out


def sinkhorn_f64(logits: np.ndarray, iters: int = 20) -> np.ndarray:
    x = np.ascontiguousarray(logits, dtype=np.float64)
    n = x.shape[-1]
    out = np.empty_like(x)
    lib().oracle_sinkhorn_f64(_p(x), _p(out), x.size // (n * n), n, iters)
    return out


def schedule(cfg: Config) -> np.ndarray:
    n = lib().oracle_num_exec(C.byref(cfg))
    if n < 0:
        raise ValueError("invalid config")
    t = np.zeros((n, 5), dtype=np.int32)
    lib().oracle_schedule(C.byref(cfg), _p(t))
    return t


def rmsnorm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(gain, dtype=np.float64)
    y = np.empty_like(x)
    lib().oracle_rmsnorm(_p(x), _p(g), _p(y), x.size // x.shape[-1], x.shape[-1], eps)
    return y


def gla_recurrent(q, k, v, g, state=None):
    q, k, v, g = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v, g))
    T, dk = q.shape
    dv = v.shape[1]
    st = np.zeros((dk, dv)) if state is None else np.array(state, dtype=np.float64)
    o = np.empty((T, dv))
    lib().oracle_gla_recurrent(_p(q), _p(k), _p(v), _p(g), _p(o), _p(st), T, dk, dv)
    return o, st


def attention_naive(q, k, v, q0=0):
    q, k, v = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v))
    o = np.empty((q.shape[0], v.shape[1]))
    lib().oracle_attention_naive(_p(q), _p(k), _p(v), _p(o), q.shape[0], k.shape[0], q0, q.shape[1])
    return o


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    y = np.array(x, dtype=np.float64)
    T, nh, d = y.shape
    p = np.ascontiguousarray(pos, dtype=np.int32)
    lib().oracle_rope(_p(y), T, nh, d, _p(p), base)
    return y


def mhc_site(s, gamma_m, phi, gain, iters=20, eps=1e-6):
    s, gm, ph, g = (np.ascontiguousarray(a, dtype=np.float64) for a in (s, gamma_m, phi, gain))
    n, H = s.shape
    coef = np.empty(2 * n + n * n)
    xh = np.empty(H)
    lib().oracle_mhc_site(_p(s), _p(gm), _p(ph), _p(g), n, H, iters, eps, _p(coef), _p(xh))
    return coef, xh


def mhc_write(s, coef, y):
    s = np.array(s, dtype=np.float64)
    coef = np.ascontiguousarray(coef, dtype=np.float64)
    y = np.ascontiguousarray(y, dtype=np.float64)
    n, H = s.shape
    lib().oracle_mhc_write(_p(s), _p(coef), _p(y), n, H)
    return s


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def attention_sublayer(cfg: Config, wq, wk, wv, wo, xh, start, kcache=None, vcache=None):
    """The model's full-attention sublayer on caller weights.  xh [B][S][hidden];
    start[b] is the position of sequence b's first token; the K/V cache slots
    [B][n_kv][max_ctx][head_dim] are updated in place (zeros if not given).
    Returns (y [B][S][hidden], kcache, vcache)."""
    xh = np.ascontiguousarray(xh, dtype=np.float64)
    B, S, H = xh.shape
    shape = (cfg.max_batch, cfg.n_kv, cfg.max_ctx, cfg.head_dim)
    kc = np.zeros(shape, np.float32) if kcache is None else kcache
    vc = np.zeros(shape, np.float32) if vcache is None else vcache
    ws = [_f32(w) for w in (wq, wk, wv, wo)]
    st = np.ascontiguousarray(start, dtype=np.int32)
    y = np.empty_like(xh)
    rc = lib().oracle_attention_sublayer(C.byref(cfg), *[_p(w) for w in ws], _p(kc), _p(vc), _p(xh), B, S,
                                         _p(st), _p(y))
    if rc != 0:
        raise ValueError("oracle_attention_sublayer failed")
    return y, kc, vc


def gla_sublayer(cfg: Config, wq, wk, wv, wg, wo, xh, state=None):
    """The model's gated-linear-attention sublayer on caller weights.  xh
    [B][S][hidden]; state [B][n_lin][d][d] (zeros if not given) is advanced.
    Returns (y [B][S][hidden], state)."""
    xh = np.ascontiguousarray(xh, dtype=np.float64)
    B, S, H = xh.shape
    st = np.zeros((B, cfg.n_lin, cfg.lin_dim, cfg.lin_dim)) if state is None else \
        np.array(state, dtype=np.float64)
    ws = [_f32(w) for w in (wq, wk, wv, wg, wo)]
    y = np.empty_like(xh)
    if lib().oracle_gla_sublayer(C.byref(cfg), *[_p(w) for w in ws], _p(st), _p(xh), B, S, _p(y)) != 0:
        raise ValueError("oracle_gla_sublayer failed")
    return y, st


def ffn_sublayer(cfg: Config, w_gate, w_up, w_down, xh):
    """The model's SwiGLU FFN on caller weights; xh [T][hidden] -> y [T][hidden]."""
    xh = np.ascontiguousarray(xh, dtype=np.float64)
    ws = [_f32(w) for w in (w_gate, w_up, w_down)]
    y = np.empty_like(xh)
    if lib().oracle_ffn_sublayer(C.byref(cfg), *[_p(w) for w in ws], _p(xh), xh.size // xh.shape[-1], _p(y)) != 0:
        raise ValueError("oracle_ffn_sublayer failed")
    return y


class Model:
    """The oracle's looped decoder with its own KV cache and linear-attention state."""

    def __init__(self, cfg: Config, seed: int = 0, weights=None):
        self.cfg = cfg
        L = lib()
        self._keep = None
        wp = None
        if weights is not None:
            arrs = [np.ascontiguousarray(w, dtype=np.float32) for w in weights]
            ptrs = (C.c_void_p * len(arrs))(*[a.ctypes.data if a.size else None for a in arrs])
            self._keep = (arrs, ptrs)
            wp = C.cast(ptrs, C.c_void_p)
        self.h = L.oracle_model_create(C.byref(cfg), seed, wp)
        if not self.h:
            raise ValueError("oracle_model_create failed")

    def close(self):
        if self.h:
            lib().oracle_model_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def num_weights(self) -> int:
        return lib().oracle_num_weights(C.byref(self.cfg))

    def weight(self, index: int) -> np.ndarray:
        n = lib().oracle_weight_numel(self.h, index)
        out = np.empty(n, dtype=np.float32)
        if n:
            lib().oracle_get_weight(self.h, index, _p(out))
        return out

    def prefill(self, tokens=None, hidden=None, all_positions=False) -> np.ndarray:
        c = self.cfg
        if c.io_mode == 0:
            tok = np.ascontiguousarray(tokens, dtype=np.int32)
            B, S = tok.shape
            rows = B * S if all_positions else B
            out = np.empty((rows, c.vocab), dtype=np.float32)
            rc = lib().oracle_prefill(self.h, _p(tok), None, B, S, _p(out), ALL_POSITIONS if all_positions else 0)
            out = out.reshape((B, S, c.vocab) if all_positions else (B, c.vocab))
        else:
            hid = np.ascontiguousarray(hidden, dtype=np.float32)
            B, S, _ = hid.shape
            out = np.empty_like(hid)
            rc = lib().oracle_prefill(self.h, None, _p(hid), B, S, _p(out), 0)
        if rc != 0:
            raise ValueError(f"oracle_prefill failed ({rc})")
        return out

    def decode_step(self, tokens) -> np.ndarray:
        tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
        out = np.empty((tok.size, self.cfg.vocab), dtype=np.float32)
        rc = lib().oracle_decode_step(self.h, _p(tok), tok.size, _p(out))
        if rc != 0:
            raise ValueError(f"oracle_decode_step failed ({rc})")
        return out

    def seq_len(self, b: int) -> int:
        return lib().oracle_seq_len(self.h, b)

    def kv(self, slot: int, B: int, length: int):
        c = self.cfg
        out = np.empty((2, B, c.n_kv, length, c.head_dim), dtype=np.float32)
        if lib().oracle_cache_read(self.h, FULL, slot, B, length, _p(out)) != 0:
            raise ValueError("bad kv slot")
        return out[0], out[1]

    def state(self, slot: int, B: int):
        c = self.cfg
        out = np.empty((B, c.n_lin, c.lin_dim, c.lin_dim), dtype=np.float32)
        if lib().oracle_cache_read(self.h, LINEAR, slot, B, 0, _p(out)) != 0:
            raise ValueError("bad state slot")
        return out

    def load_kv(self, slot: int, k: np.ndarray, v: np.ndarray):
        """Test-only: write K and V [B][n_kv][len][head_dim] into a KV slot."""
        k, v = _f32(k), _f32(v)
        B, _, length, _ = k.shape
        buf = np.ascontiguousarray(np.stack([k, v]))
        if lib().oracle_cache_write(self.h, FULL, slot, B, length, _p(buf)) != 0:
            raise ValueError("bad kv slot")

    def load_state(self, slot: int, state: np.ndarray):
        """Test-only: write the state [B][n_lin][d][d] of a linear slot."""
        s = _f32(state)
        if lib().oracle_cache_write(self.h, LINEAR, slot, s.shape[0], 0, _p(s)) != 0:
            raise ValueError("bad state slot")

    def set_seq_len(self, b: int, length: int):
        if lib().oracle_set_seq_len(self.h, b, length) != 0:
            raise ValueError("bad sequence or length")

    def set_weight(self, index: int, values: np.ndarray):
        """Test-only: replace weight tensor `index` (canonical order)."""
        x = _f32(values)
        if x.size != lib().oracle_weight_numel(self.h, index) or lib().oracle_set_weight(self.h, index, _p(x)) != 0:
            raise ValueError("bad weight index or size")
