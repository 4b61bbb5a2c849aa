"""mhc_prologue_noalloc, the variant of the mHC read site for callers that
cannot allocate device memory (a runtime whose pool owns every device
allocation, or a path that cannot afford cudaMalloc's implicit sync): it must
give the same results as mhc_prologue with a caller scratch buffer, on two
calls in a row that share the library's fixed scratch array.

This file is collected last so that a run stopping at the first failure has
already run every other test."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import looped_weight_shared_b200 as L  # noqa: E402

pytestmark = pytest.mark.gpu


def make(T, H, seed):
    g = torch.Generator().manual_seed(seed)
    s = torch.randn(2, T, H, generator=g)
    gamma = 0.5 + torch.rand(2 * H, generator=g)
    phi = 0.02 * torch.randn(8, 2 * H, generator=g)
    gain = 0.5 + torch.rand(H, generator=g)
    return [x.cuda() for x in (s, gamma, phi, gain)]


def with_scratch(s, gamma, phi, gain, dtype):
    T, H = s.shape[1], s.shape[2]
    coef = torch.empty(T, 8, device="cuda")
    xh = torch.empty(T, H, device="cuda", dtype=dtype)
    L.mhc_prologue(s, gamma, phi, gain, coef, xh, torch.empty(18 * T, device="cuda"))
    return coef, xh


def without_scratch(s, gamma, phi, gain, dtype):
    T, H = s.shape[1], s.shape[2]
    coef = torch.full((T, 8), float("nan"), device="cuda")
    xh = torch.full((T, H), float("nan"), device="cuda").to(dtype)
    L.mhc_prologue_noalloc(s, gamma, phi, gain, coef, xh)
    return coef, xh


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_the_scratch_entry_point_twice(dtype):
    # two calls in a row with different inputs: the second must not see the first's leftovers
    for T, H, seed in ((4096, 4096, 1), (777, 512, 2)):
        args = make(T, H, seed)
        ref_c, ref_x = with_scratch(*args, dtype)
        got_c, got_x = without_scratch(*args, dtype)
        torch.cuda.synchronize()
        np.testing.assert_allclose(got_c.cpu().numpy(), ref_c.cpu().numpy(), rtol=2e-5, atol=2e-6)
        np.testing.assert_allclose(got_x.float().cpu().numpy(), ref_x.float().cpu().numpy(), rtol=2e-5, atol=2e-5)
    assert L.loop_device_status() == 0


def test_noalloc_rejects_more_tokens_than_its_scratch():
    T, H = 65537, 4
    s = torch.zeros(2, T, H, device="cuda")
    z = torch.ones(2 * H * 8, device="cuda")
    with pytest.raises(L.LoopError) as e:
        L.mhc_prologue_noalloc(s, z, z, z, torch.empty(T, 8, device="cuda"), torch.empty(T, H, device="cuda"))
    assert e.value.code == L.LOOP_ERANGE
    assert "65536" in L.last_error()
