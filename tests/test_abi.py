"""CPU checks of the C ABI: the library loads, exports every entry point the
public headers declare, and its host-side bookkeeping (execution table,
weight count, argument checks) matches the oracle bit for bit."""

import glob
import os
import re

import numpy as np
import pytest

import oracle
import looped_weight_shared_b200 as L
from seeded import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"LOOP_API\s+[\w\s\*]+?\b(\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert {"loop_model_create", "loop_prefill", "loop_decode_step", "mhc_sinkhorn", "loop_model_destroy"} <= names
    lib = L.lib()
    for n in sorted(names):
        assert hasattr(lib, n), n
    assert set(L.API) == names


@pytest.mark.parametrize("name,over", [
    ("loop9b_prefill_b4_s8192", {}),
    ("tiny_fp32", {}),
    ("group9b_s4096", {}),
    ("loop9b_prefill_b4_s8192", {"n_loops": 3}),
    ("tiny_fp32", {"n_loops": 1, "n_block": 8}),
    ("tiny_fp32", {"n_prelude": 0, "n_coda": 8}),
])
def test_schedule_bit_exact_vs_oracle(name, over):
    m = dict(W.model_config(name, **over), max_batch=2, max_ctx=16)
    a = L.loop_schedule(L.make_config(**m))
    b = oracle.schedule(oracle.make_config(**m))
    np.testing.assert_array_equal(a, b)
    assert L.loop_num_weights(L.make_config(**m)) == oracle.lib().oracle_num_weights(
        __import__("ctypes").byref(oracle.make_config(**m)))


@pytest.mark.parametrize("bad", [
    {"n_block": 5}, {"n_prelude": 2}, {"n_q": 6, "n_kv": 4}, {"head_dim": 7}, {"max_batch": 0},
    {"dtype": 3}, {"group": 0}, {"full_slot": 4}, {"n_loops": 0},
])
def test_invalid_configs_rejected(bad):
    m = dict(W.model_config("tiny_fp32"), max_batch=1, max_ctx=8)
    m.update(bad)
    with pytest.raises(L.LoopError) as e:
        L.loop_num_exec(L.make_config(**m))
    assert e.value.code == L.LOOP_EINVAL


def test_create_rejects_without_touching_the_device():
    m = dict(W.model_config("tiny_fp32"), max_batch=1, max_ctx=8, n_streams=3)
    with pytest.raises(L.LoopError) as e:
        L.loop_model_create(L.make_config(**m))
    assert e.value.code == L.LOOP_EUNSUPPORTED
    m["n_streams"] = 2
    m["n_block"] = 6
    with pytest.raises(L.LoopError) as e:
        L.loop_model_create(L.make_config(**m))
    assert e.value.code == L.LOOP_EINVAL
    assert "invalid" in L.last_error()


def test_entry_points_reject_null_without_touching_the_device():
    """Argument errors return a status before any device work, including for
    the append and ragged-prefill entry points."""
    lib = L.lib()
    assert lib.loop_prefill(None, None, None, 1, 1, None, 0, None) == L.LOOP_EINVAL
    assert lib.loop_decode_step(None, None, 1, None, None) == L.LOOP_EINVAL
    assert lib.loop_extend(None, None, 1, 1, None, 0, None) == L.LOOP_EINVAL
    assert lib.loop_prefill_ragged(None, None, None, 0, 1, None, 0, None) == L.LOOP_EINVAL
    assert "NULL" in L.last_error()
    assert lib.mhc_sinkhorn(None, None, 1, 2, 20, None) == L.LOOP_EINVAL
