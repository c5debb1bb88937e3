"""The tcgen05 GEMM engine on its own, against a library matmul in fp64.

Covers both operand majors, bf16 (kind::f16) and fp32-as-tf32 (kind::tf32),
ragged M/N/K tails, batching and split-K, at sizes spanning several tiles.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


CASES = [
    # eb, a_mn, b_mn, bn, M, N, K, batches, splits
    (2, 0, 0, 128, 128, 128, 64, 1, 1),
    (2, 0, 0, 128, 256, 256, 256, 2, 1),
    (2, 0, 0, 256, 200, 264, 328, 3, 1),
    (2, 0, 0, 64, 136, 72, 136, 1, 2),
    (2, 1, 0, 128, 256, 128, 192, 2, 1),
    (2, 0, 1, 128, 256, 128, 192, 2, 1),
    (2, 1, 1, 128, 256, 256, 448, 2, 3),
    (2, 1, 1, 256, 384, 512, 1000, 1, 4),
    (2, 1, 1, 64, 192, 64, 6084, 2, 5),
    (4, 0, 0, 128, 128, 128, 64, 1, 1),
    (4, 0, 0, 256, 256, 256, 300, 2, 1),
    (4, 0, 0, 128, 384, 256, 1000, 2, 3),
]
# fp32-as-tf32 operands are K-major only: an MN-major tf32 operand gave wrong
# products on this toolchain, so the engine rejects that combination.


@pytest.mark.parametrize("eb,a_mn,b_mn,bn,M,N,K,batches,splits", CASES)
def test_tc_gemm_matches_matmul(eb, a_mn, b_mn, bn, M, N, K, batches, splits):
    from weight_sequence_mixing_b200 import binding

    g = torch.Generator().manual_seed(M * 7 + N * 3 + K + eb)
    dt = torch.bfloat16 if eb == 2 else torch.float32
    a = torch.randn((batches, M, K), generator=g).to(dt)  # logical A [z][m][k]
    b = torch.randn((batches, N, K), generator=g).to(dt)  # logical B [z][n][k]
    A = (a.transpose(1, 2) if a_mn else a).contiguous().cuda()
    B = (b.transpose(1, 2) if b_mn else b).contiguous().cuda()
    C = binding.selftest_gemm(A, B, eb, a_mn, b_mn, bn, M, N, K, batches, splits)
    torch.cuda.synchronize()
    got = C.double().sum(0).cpu()
    ref = torch.matmul(a.double(), b.double().transpose(1, 2))
    err = ((got - ref).norm() / ref.norm()).item()
    tol = 1e-5 if eb == 2 else 3e-3
    assert torch.isfinite(got).all()
    assert err < tol, f"relative Frobenius error {err:.3e}"
