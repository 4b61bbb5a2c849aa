"""The fused mHC prologue (coefficients, Sinkhorn, stream read, RMSNorm)
through the C ABI against the oracle's per-token mHC site."""

import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
import looped_weight_shared_b200 as L  # noqa: E402

pytestmark = pytest.mark.gpu


def inputs(T, H, seed, phi_scale=0.02):
    rng = np.random.default_rng(seed)
    s = rng.normal(0, 1, size=(2, T, H)).astype(np.float32)
    s[1] += rng.normal(0, 0.5, size=(T, H)).astype(np.float32)
    gamma = rng.uniform(0.5, 1.5, size=2 * H).astype(np.float32)
    phi = rng.normal(0, phi_scale, size=(8, 2 * H)).astype(np.float32)
    gain = rng.uniform(0.5, 1.5, size=H).astype(np.float32)
    return s, gamma, phi, gain


def run_gpu(s, gamma, phi, gain, out_dtype):
    T, H = s.shape[1], s.shape[2]
    coef = torch.empty((T, 8), device="cuda")
    xh = torch.empty((T, H), device="cuda", dtype=out_dtype)
    scratch = torch.full((18 * T,), float("nan"), device="cuda")
    L.mhc_prologue(torch.from_numpy(s).cuda(), torch.from_numpy(gamma).cuda(), torch.from_numpy(phi).cuda(),
                   torch.from_numpy(gain).cuda(), coef, xh, scratch)
    torch.cuda.synchronize()
    return coef.cpu().numpy(), xh.float().cpu().numpy()


@pytest.mark.parametrize("T,H", [(1, 256), (67, 512), (300, 4096), (9, 6144)])
def test_mhc_prologue_matches_oracle(T, H):
    s, gamma, phi, gain = inputs(T, H, T + H)
    coef, xh = run_gpu(s, gamma, phi, gain, torch.float32)
    for t in range(T):
        c_ref, x_ref = oracle.mhc_site(s[:, t], gamma, phi, gain, iters=20, eps=1e-6)
        np.testing.assert_allclose(coef[t], c_ref, rtol=2e-5, atol=2e-6)
        np.testing.assert_allclose(xh[t], x_ref, rtol=2e-5, atol=2e-5)
    # bf16 output: the same values rounded
    _, xb = run_gpu(s, gamma, phi, gain, torch.bfloat16)
    assert np.abs(xb - xh).max() <= np.abs(xh).max() * 2**-8


def test_mhc_prologue_large_logits_and_columns():
    """Phi large enough that the cross ratio of the mixing logits is far from 0:
    columns of H_res still sum to 1 and rows follow the 2x2 closed form."""
    T, H = 40, 1024
    s, gamma, phi, gain = inputs(T, H, 3, phi_scale=0.2)
    coef, _ = run_gpu(s, gamma, phi, gain, torch.float32)
    res = coef[:, 4:].reshape(T, 2, 2)
    np.testing.assert_allclose(res.sum(axis=1), 1.0, atol=4 * 2**-24)
    # sigmoid saturates to exactly 0 or 1 in fp32 at these logits
    assert np.all((coef[:, :2] >= 0) & (coef[:, :2] <= 1)) and np.all((coef[:, 2:4] >= 0) & (coef[:, 2:4] <= 2))
    for t in range(T):
        c_ref, _ = oracle.mhc_site(s[:, t], gamma, phi, gain, iters=20, eps=1e-6)
        np.testing.assert_allclose(coef[t], c_ref, rtol=5e-5, atol=5e-6)


def test_mhc_prologue_rejects_bad_shapes():
    z = torch.zeros(64, device="cuda")
    with pytest.raises(L.LoopError):
        L.lib().mhc_prologue  # exists
        L.mhc_prologue(torch.zeros((2, 1, 6), device="cuda"), z, z, z, torch.zeros((1, 8), device="cuda"),
                       torch.zeros((1, 6), device="cuda"), z)
