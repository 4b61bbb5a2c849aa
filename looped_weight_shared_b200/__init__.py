"""Python binding of the looped-decoder C ABI (include/looped.h).

Argument marshalling only: every step of the forward pass runs in the CUDA
library ``_looped.so`` built from ``csrc/`` (see ``build.py``).  There is no
fallback: if the library is missing or cannot load, importing the functions
below raises.  torch supplies device memory and the current CUDA stream.
"""

from __future__ import annotations

import ctypes as C
import os

_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_DIR, "_looped.so")

LOOP_OK, LOOP_EINVAL, LOOP_ENOMEM, LOOP_ECUDA, LOOP_ERANGE, LOOP_EUNSUPPORTED, LOOP_ETIMEOUT = 0, -1, -2, -3, -4, -5, -6
LOOP_F32, LOOP_BF16 = 0, 1
LOOP_TOKENS_TO_LOGITS, LOOP_HIDDEN_TO_HIDDEN = 0, 1
LOOP_ALL_POSITIONS = 1
LOOP_KIND_LINEAR, LOOP_KIND_FULL = 0, 1
LOOP_K_GEMM, LOOP_K_ATTENTION, LOOP_K_LINEAR_ATTENTION, LOOP_K_MHC, LOOP_K_NORM, LOOP_K_OTHER = range(6)
KERNEL_CLASSES = ("gemm", "attention", "linear_attention", "mhc", "norm", "other")

API = ("loop_num_exec", "loop_schedule", "loop_num_weights", "loop_model_create", "loop_prefill",
       "loop_decode_step", "mhc_sinkhorn", "loop_model_destroy", "loop_seq_len", "loop_cache_read",
       "loop_weight_read", "loop_device_status", "loop_clear_device_status", "loop_last_error",
       "loop_gemm_bf16", "loop_set_timing", "loop_timing_read", "loop_launch_count", "mhc_prologue",
       "mhc_prologue_noalloc", "loop_selftest_timeout", "loop_extend", "loop_prefill_ragged", "loop_capture")


class loop_config(C.Structure):
    _fields_ = [(n, C.c_int32) for n in (
        "n_prelude", "n_block", "n_loops", "n_coda", "group", "full_slot", "hidden", "ffn", "vocab",
        "n_q", "n_kv", "head_dim", "n_lin", "lin_dim", "lin_chunk", "n_streams", "sinkhorn_iters")] + [
        ("rope_base", C.c_float), ("norm_eps", C.c_float)] + [
        (n, C.c_int32) for n in ("dtype", "io_mode", "max_batch", "max_ctx", "kv_pages")]


def make_config(**kw) -> loop_config:
    c = loop_config()
    for k, v in kw.items():
        setattr(c, k, v)
    return c


class LoopError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed with status {code}: {last_error()}")
        self.code = code


_lib = None


def lib():
    """Load the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m looped_weight_shared_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, vp, i32, u32, u64 = C.POINTER, C.c_void_p, C.c_int32, C.c_uint32, C.c_uint64
        sig = {
            "loop_num_exec": (i32, [P(loop_config)]),
            "loop_schedule": (i32, [P(loop_config), vp]),
            "loop_num_weights": (i32, [P(loop_config)]),
            "loop_model_create": (i32, [P(loop_config), vp, u64, P(vp)]),
            "loop_prefill": (i32, [vp, vp, vp, i32, i32, vp, u32, vp]),
            "loop_decode_step": (i32, [vp, vp, i32, vp, vp]),
            "loop_extend": (i32, [vp, vp, i32, i32, vp, u32, vp]),
            "loop_prefill_ragged": (i32, [vp, vp, vp, i32, i32, vp, u32, vp]),
            "mhc_sinkhorn": (i32, [vp, vp, i32, i32, i32, vp]),
            "loop_model_destroy": (None, [vp]),
            "loop_seq_len": (i32, [vp, i32]),
            "loop_cache_read": (i32, [vp, i32, i32, i32, i32, vp, vp]),
            "loop_weight_read": (i32, [vp, i32, vp, vp]),
            "loop_device_status": (i32, []),
            "loop_clear_device_status": (None, []),
            "loop_last_error": (C.c_char_p, []),
            "loop_gemm_bf16": (i32, [vp, vp, C.c_int64, C.c_int64, C.c_int64, vp, C.c_int64, i32, vp]),
            "loop_set_timing": (i32, [vp, i32]),
            "loop_timing_read": (i32, [vp, i32, P(C.c_double), P(C.c_int64), P(C.c_double), i32]),
            "loop_launch_count": (C.c_int64, [vp]),
            "mhc_prologue": (i32, [vp, C.c_int64, i32, vp, vp, vp, i32, C.c_float, vp, vp, i32, vp, vp]),
            "mhc_prologue_noalloc": (i32, [vp, C.c_int64, i32, vp, vp, vp, i32, C.c_float, vp, vp, i32, vp]),
            "loop_selftest_timeout": (i32, [i32]),
            "loop_capture": (i32, [vp, i32, i32, i32, vp, vp, vp, vp, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def last_error() -> str:
    return lib().loop_last_error().decode()


def _check(fn: str, rc: int) -> int:
    if rc < 0:
        raise LoopError(fn, rc)
    return rc


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return C.c_void_p(stream if isinstance(stream, int) else stream.cuda_stream)


# ---- the C ABI, one function per entry point ----

def loop_num_exec(cfg: loop_config) -> int:
    return _check("loop_num_exec", lib().loop_num_exec(C.byref(cfg)))


def loop_schedule(cfg: loop_config):
    import numpy as np
    n = loop_num_exec(cfg)
    t = np.zeros((n, 5), dtype=np.int32)
    _check("loop_schedule", lib().loop_schedule(C.byref(cfg), t.ctypes.data_as(C.c_void_p)))
    return t


def loop_num_weights(cfg: loop_config) -> int:
    return _check("loop_num_weights", lib().loop_num_weights(C.byref(cfg)))


def loop_model_create(cfg: loop_config, host_weights=None, seed: int = 0) -> int:
    """Returns the opaque model handle.  host_weights: list of contiguous fp32
    numpy arrays in the canonical order (None entries for empty tensors)."""
    import numpy as np
    wp = None
    keep = None
    if host_weights is not None:
        arrs = [None if w is None else np.ascontiguousarray(w, dtype=np.float32) for w in host_weights]
        ptrs = (C.c_void_p * len(arrs))(*[None if a is None or a.size == 0 else a.ctypes.data for a in arrs])
        keep = (arrs, ptrs)
        wp = C.cast(ptrs, C.c_void_p)
    h = C.c_void_p()
    _check("loop_model_create", lib().loop_model_create(C.byref(cfg), wp, seed, C.byref(h)))
    del keep
    return h.value


def loop_prefill(model: int, tokens=None, hidden=None, out=None, flags: int = 0, stream=None) -> None:
    """tokens: int32 cuda [B, S] or hidden: fp32 cuda [B, S, H]; out: fp32 cuda."""
    x = tokens if tokens is not None else hidden
    B, S = int(x.shape[0]), int(x.shape[1])
    _check("loop_prefill", lib().loop_prefill(C.c_void_p(model), _ptr(tokens), _ptr(hidden), B, S, _ptr(out),
                                              flags, _stream(stream)))


def loop_decode_step(model: int, tokens, logits, stream=None) -> None:
    """tokens: int32 cuda [B]; logits: fp32 cuda [B, vocab]."""
    _check("loop_decode_step", lib().loop_decode_step(C.c_void_p(model), _ptr(tokens), int(tokens.shape[0]),
                                                      _ptr(logits), _stream(stream)))


def loop_extend(model: int, tokens, out, flags: int = 0, stream=None) -> None:
    """tokens: int32 cuda [B, k] appended to each sequence; out: fp32 cuda
    [B, vocab] (last appended position) or [B, k, vocab] with LOOP_ALL_POSITIONS."""
    B, k = int(tokens.shape[0]), int(tokens.shape[1])
    _check("loop_extend", lib().loop_extend(C.c_void_p(model), _ptr(tokens), B, k, _ptr(out), flags,
                                            _stream(stream)))


def loop_prefill_ragged(model: int, tokens, lens, out, b0: int = 0, flags: int = 0, stream=None) -> None:
    """tokens: int32 cuda, the sequences packed one after another; lens: their
    lengths (host ints); prefills sequences b0 .. b0 + len(lens) - 1 only.
    out: fp32 cuda [len(lens), vocab], or [sum(lens), vocab] with LOOP_ALL_POSITIONS."""
    import numpy as np
    arr = np.ascontiguousarray(np.asarray(lens, dtype=np.int32))
    _check("loop_prefill_ragged", lib().loop_prefill_ragged(C.c_void_p(model), _ptr(tokens),
                                                            arr.ctypes.data_as(C.c_void_p), int(b0), int(arr.size),
                                                            _ptr(out), flags, _stream(stream)))


def mhc_sinkhorn(logits, out, iters: int = 20, stream=None) -> None:
    """logits, out: fp32 cuda [count, n, n]."""
    n = int(logits.shape[-1])
    count = logits.numel() // (n * n)
    _check("mhc_sinkhorn", lib().mhc_sinkhorn(_ptr(logits), _ptr(out), count, n, iters, _stream(stream)))


def loop_model_destroy(model: int) -> None:
    lib().loop_model_destroy(C.c_void_p(model))


def loop_seq_len(model: int, b: int) -> int:
    return _check("loop_seq_len", lib().loop_seq_len(C.c_void_p(model), b))


def loop_cache_read(model: int, kind: int, slot: int, B: int, length: int, out, stream=None) -> None:
    _check("loop_cache_read", lib().loop_cache_read(C.c_void_p(model), kind, slot, B, length, _ptr(out),
                                                    _stream(stream)))


def loop_capture(model: int, exec_: int, head0: int = 0, nheads: int = 1, q=None, k=None, v=None, gate=None,
                 o=None) -> None:
    """Arm a capture of execution exec_'s attention inputs and output (see
    include/looped.h); exec_ < 0 disarms every capture."""
    _check("loop_capture", lib().loop_capture(C.c_void_p(model), exec_, head0, nheads, _ptr(q), _ptr(k), _ptr(v),
                                              _ptr(gate), _ptr(o)))


def loop_weight_read(model: int, index: int, out, stream=None) -> None:
    _check("loop_weight_read", lib().loop_weight_read(C.c_void_p(model), index, _ptr(out), _stream(stream)))


def loop_device_status() -> int:
    return lib().loop_device_status()


def loop_clear_device_status() -> None:
    lib().loop_clear_device_status()


STATUS_WAIT_PRODUCER, STATUS_WAIT_MMA, STATUS_WAIT_EPILOGUE, STATUS_WAIT_OTHER = 1, 2, 4, 8
STATUS_BAD_TOKEN, STATUS_SELFTEST = 16, 32


def loop_selftest_timeout(timeout_ms: int = 50) -> int:
    return _check("loop_selftest_timeout", lib().loop_selftest_timeout(timeout_ms))


def loop_gemm_bf16(A, W, C_out, use_tensor_cores: bool = True, stream=None) -> None:
    """C_out[M, N] fp32 = A[M, K] @ W[N, K].T for bf16 cuda tensors."""
    M, K = int(A.shape[0]), int(A.shape[1])
    N = int(W.shape[0])
    _check("loop_gemm_bf16", lib().loop_gemm_bf16(_ptr(A), _ptr(W), M, N, K, _ptr(C_out), int(C_out.stride(0)),
                                                  1 if use_tensor_cores else 0, _stream(stream)))


def loop_set_timing(model: int, enable: bool) -> None:
    _check("loop_set_timing", lib().loop_set_timing(C.c_void_p(model), 1 if enable else 0))


def loop_timing_read(model: int, cls: int, reset: bool = False):
    """(total_ms, launches, work) of kernel class cls."""
    ms, n, w = C.c_double(), C.c_int64(), C.c_double()
    _check("loop_timing_read", lib().loop_timing_read(C.c_void_p(model), cls, C.byref(ms), C.byref(n), C.byref(w),
                                                      1 if reset else 0))
    return ms.value, n.value, w.value


def loop_launch_count(model: int) -> int:
    return lib().loop_launch_count(C.c_void_p(model))


def mhc_prologue(streams, gamma, phi, gain, coef, xhat, scratch, iters: int = 20, eps: float = 1e-6,
                 stream=None) -> None:
    """streams fp32 cuda [2, T, H]; coef fp32 [T, 8]; xhat fp32 or bf16 [T, H]; scratch fp32 >= 18 T."""
    import torch
    T, H = int(streams.shape[1]), int(streams.shape[2])
    dt = LOOP_BF16 if xhat.dtype == torch.bfloat16 else LOOP_F32
    _check("mhc_prologue", lib().mhc_prologue(_ptr(streams), T, H, _ptr(gamma), _ptr(phi), _ptr(gain), iters, eps,
                                              _ptr(coef), _ptr(xhat), dt, _ptr(scratch), _stream(stream)))


def mhc_prologue_noalloc(streams, gamma, phi, gain, coef, xhat, iters: int = 20, eps: float = 1e-6,
                         stream=None) -> None:
    """mhc_prologue without a scratch argument: for callers that cannot
    allocate device memory (the library's fixed scratch array is used)."""
    import torch
    T, H = int(streams.shape[1]), int(streams.shape[2])
    dt = LOOP_BF16 if xhat.dtype == torch.bfloat16 else LOOP_F32
    _check("mhc_prologue_noalloc", lib().mhc_prologue_noalloc(_ptr(streams), T, H, _ptr(gamma), _ptr(phi),
                                                              _ptr(gain), iters, eps, _ptr(coef), _ptr(xhat), dt,
                                                              _stream(stream)))
