"""Failure detection without a GPU fault: a bounded device wait that runs
out, out-of-range token ids, and calls rejected on the host before any
launch."""

import numpy as np
import pytest

from seeded import workloads as W

torch = pytest.importorskip("torch")
import looped_weight_shared_b200 as L  # noqa: E402

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    L.loop_clear_device_status()
    st = L.loop_selftest_timeout(50)
    assert st & L.STATUS_SELFTEST
    L.loop_clear_device_status()
    assert L.loop_device_status() == 0
    x = torch.ones(1000, device="cuda")  # the context is still usable
    assert float(x.sum()) == 1000.0


def test_bad_token_ids_flag_the_status_word():
    m = dict(W.model_config("tiny_fp32"), max_batch=1, max_ctx=8)
    g = L.loop_model_create(L.make_config(**m), seed=0)
    try:
        L.loop_clear_device_status()
        out = torch.empty((1, m["vocab"]), device="cuda")
        L.loop_prefill(g, tokens=torch.tensor([[1, m["vocab"], 2]], dtype=torch.int32, device="cuda"), out=out)
        assert L.loop_device_status() & L.STATUS_BAD_TOKEN
        L.loop_clear_device_status()
        L.loop_prefill(g, tokens=torch.tensor([[1, 5, 2]], dtype=torch.int32, device="cuda"), out=out)
        assert L.loop_device_status() == 0 and torch.isfinite(out).all()
    finally:
        L.loop_model_destroy(g)


def test_host_rejections_launch_nothing():
    m = dict(W.model_config("tiny_fp32"), max_batch=2, max_ctx=8)
    g = L.loop_model_create(L.make_config(**m), seed=0)
    try:
        n0 = L.loop_launch_count(g)
        out = torch.empty((2, m["vocab"]), device="cuda")
        for tok, code in ((torch.zeros((0, 4), dtype=torch.int32, device="cuda"), L.LOOP_EINVAL),
                          (torch.zeros((3, 4), dtype=torch.int32, device="cuda"), L.LOOP_ERANGE),
                          (torch.zeros((1, 9), dtype=torch.int32, device="cuda"), L.LOOP_ERANGE)):
            with pytest.raises(L.LoopError) as e:
                L.loop_prefill(g, tokens=tok, out=out)
            assert e.value.code == code
        with pytest.raises(L.LoopError) as e:
            L.mhc_sinkhorn(torch.zeros((4, 9, 9), device="cuda"), torch.zeros((4, 9, 9), device="cuda"))
        assert e.value.code == L.LOOP_EINVAL
        assert L.loop_launch_count(g) == n0
        with pytest.raises(L.LoopError) as e:
            L.loop_selftest_timeout(0)
        assert e.value.code == L.LOOP_EINVAL
    finally:
        L.loop_model_destroy(g)
