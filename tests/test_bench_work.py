"""The algorithmic work bench.py divides by, checked against the per-layer
parameter counts and per-token FLOP and per-step byte figures derived
independently from the model's shapes (hidden 4096, FFN 12288, GQA 32/8 x
128, 32 GLA heads x 128, vocabulary 248,320, 4 + 24 x 2 + 4 executions)."""

import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from seeded import workloads as W  # noqa: E402


def _m(name):
    return dict(W.WORKLOADS[name]["model"])


def test_layer_matrix_parameters():
    m = _m("loop9b_prefill_b4_s8192")
    # linear: q, k, v (3 x 4096) + gate (32) rows of 4096, o 4096 x 4096, SwiGLU 3 x 4096 x 12288
    assert bench.layer_weight_bytes(m, False) // 2 == 218_234_880
    # full: q (4096) + k, v (2 x 1024) rows of 4096, o, SwiGLU
    assert bench.layer_weight_bytes(m, True) // 2 == 192_937_984


def test_prefill_flops_9b():
    w = W.WORKLOADS["loop9b_prefill_b4_s8192"]
    f = bench.prefill_step_flops(_m("loop9b_prefill_b4_s8192"), w["batch"], w["seq"])
    T = w["batch"] * w["seq"]
    assert f["projections"] / T / 1e9 == pytest.approx(23.73, abs=0.01)
    assert f["attention"] / T / 1e9 == pytest.approx(0.94, abs=0.01)
    assert f["linear_attention"] / T / 1e9 == pytest.approx(0.13, abs=0.01)
    assert f["lm_head"] == 2 * 4 * 4096 * 248320
    assert f["total"] / 1e15 == pytest.approx(0.813, abs=0.001)


def test_prefill_flops_262k():
    w = W.WORKLOADS["loop9b_prefill_b1_s262144"]
    f = bench.prefill_step_flops(_m("loop9b_prefill_b1_s262144"), w["batch"], w["seq"])
    assert f["total"] / 1e15 == pytest.approx(14.14, rel=0.005)
    assert f["attention"] / f["total"] == pytest.approx(0.558, abs=0.005)


def test_decode_bytes_9b():
    w = W.WORKLOADS["loop9b_decode_b64_ctx32768"]
    b = bench.decode_step_bytes(_m("loop9b_decode_b64_ctx32768"), w["batch"], w["seq"])
    assert b["weights"] / 1e9 == pytest.approx(25.77, abs=0.01)
    assert b["kv"] / 1e9 == pytest.approx(120.26, abs=0.05)
    assert b["state"] / 1e9 == pytest.approx(11.27, abs=0.01)
    assert b["total"] / 1e9 == pytest.approx(157.3, abs=0.1)
