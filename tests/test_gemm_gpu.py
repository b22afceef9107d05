"""Unit parity of the tcgen05/TMA GEMM through the C ABI (mgt_gemm_bf16): every combination of
K-major / MN-major operands, ragged M, N and K (tile tails, K shorter than one k-tile), against
the plain definition C = A B^T evaluated in float64 on the CPU."""
import pytest
import torch

import tensor_transformer_layer_megatron_b200 as mgt

pytestmark = pytest.mark.gpu


def ceil8(v):
    return (v + 7) // 8 * 8


# For K-major B, (2048, 12288, 64) selects the 224-wide pair tile and (2048, 3000, 72) the
# 192-wide one with N ragged inside the last tile; the others take 128 or 256.
SHAPES = [(128, 256, 64), (200, 300, 136), (1, 8, 8), (1000, 520, 1000), (256, 384, 4096),
          (129, 129, 72), (2048, 12288, 64), (1000, 4096, 200), (2048, 3000, 72)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_gemm_bf16(M, N, K, a_mn, b_mn):
    g = torch.Generator().manual_seed(M * 7919 + N * 31 + K + 2 * a_mn + b_mn)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    # storage with leading dimensions padded to multiples of 8 elements
    if a_mn:
        lda = ceil8(M)
        As = torch.zeros(K, lda, dtype=torch.bfloat16); As[:, :M] = A.T
    else:
        lda = ceil8(K)
        As = torch.zeros(M, lda, dtype=torch.bfloat16); As[:, :K] = A
    if b_mn:
        ldb = ceil8(N)
        Bs = torch.zeros(K, ldb, dtype=torch.bfloat16); Bs[:, :N] = B.T
    else:
        ldb = ceil8(K)
        Bs = torch.zeros(N, ldb, dtype=torch.bfloat16); Bs[:, :K] = B
    ldc = (N + 3) // 4 * 4
    dA, dB = As.cuda(), Bs.cuda()
    C = torch.full((M, ldc), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mgt.gemm_bf16(dA, dB, C, M, N, K, a_mn, b_mn, lda, ldb, ldc, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A.double() @ B.double().T
    got = C[:, :N].double().cpu()
    err = (got - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5, err
    assert torch.isnan(C[:, N:]).all()  # nothing written past N
