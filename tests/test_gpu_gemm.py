"""The projection GEMM (tcgen05 and CUDA-core kernels) against an fp64 matrix
product of the same bf16 operands, through the C ABI."""

import numpy as np
import pytest

from metrics import rel_err

torch = pytest.importorskip("torch")
import looped_weight_shared_b200 as L  # noqa: E402

pytestmark = pytest.mark.gpu


def operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16)
    ref = (A.double() @ W.double().T).numpy()
    return A.cuda(), W.cuda(), ref


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (200, 512, 256), (333, 1000, 512), (1024, 4096, 4096),
                                   (130, 12320, 4096), (4096, 6144, 4096), (77, 24576, 128)])
def test_tc_gemm_matches_fp64(M, N, K):
    A, W, ref = operands(M, N, K, M * 7 + N + K)
    C = torch.full((M, N), float("nan"), device="cuda")
    L.loop_gemm_bf16(A, W, C, use_tensor_cores=True)
    torch.cuda.synchronize()
    got = C.cpu().numpy()
    assert np.isfinite(got).all()
    assert rel_err(got, ref) < 2e-5
    assert L.loop_device_status() == 0


def test_tc_gemm_deterministic_and_matches_simt():
    A, W, ref = operands(517, 2048, 1024, 3)
    C1 = torch.empty(517, 2048, device="cuda")
    C2 = torch.empty_like(C1)
    C3 = torch.empty_like(C1)
    L.loop_gemm_bf16(A, W, C1, use_tensor_cores=True)
    L.loop_gemm_bf16(A, W, C2, use_tensor_cores=True)
    L.loop_gemm_bf16(A, W, C3, use_tensor_cores=False)
    torch.cuda.synchronize()
    assert torch.equal(C1, C2)
    assert rel_err(C3.cpu().numpy(), ref) < 2e-5
    assert rel_err(C1.cpu().numpy(), C3.cpu().numpy()) < 2e-5


def test_tc_gemm_row_stride_and_rejects_bad_k():
    A, W, ref = operands(64, 256, 192, 5)
    C = torch.zeros(64, 300, device="cuda")
    L.loop_gemm_bf16(A, W, C[:, :256], use_tensor_cores=True)
    torch.cuda.synchronize()
    assert rel_err(C[:, :256].cpu().numpy(), ref) < 2e-5
    assert torch.count_nonzero(C[:, 256:]) == 0
    A2 = torch.zeros(8, 100, dtype=torch.bfloat16, device="cuda")
    W2 = torch.zeros(256, 100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LoopError) as e:
        L.loop_gemm_bf16(A2, W2, torch.empty(8, 256, device="cuda"))
    assert e.value.code == L.LOOP_EUNSUPPORTED
