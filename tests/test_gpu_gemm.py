"""The library's GEMMs in isolation: C = A B^T with bf16 operands and fp32
accumulation, tcgen05 tensor-core path and CUDA-core path, against torch's
fp32 product of the same bf16 values (ragged M, N and K tails included)."""
import pytest
import torch

import zeroth_order_transformer_dust_b200 as dust

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx(cuda_ok):
    return dust.Context(0)


SHAPES = [(128, 256, 64), (256, 512, 128), (300, 500, 72), (1, 16, 8), (129, 257, 1032),
          (1000, 50304, 64), (2048, 1024, 1024), (4096, 3072, 768), (64, 768, 3072)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("path", [2, 1])
def test_gemm_matches_fp32_product(ctx, M, N, K, path):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N * 3 + K)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    C = ctx.debug_gemm(A, B, path=path)
    ref = A.float() @ B.float().T
    err = ((C - ref).norm() / ref.norm()).item()
    assert err < 1e-5, err


def test_tensor_core_path_rejects_unaligned_k(ctx):
    A = torch.zeros(128, 30, device="cuda", dtype=torch.bfloat16)
    B = torch.zeros(128, 30, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(dust.DustError) as ei:
        ctx.debug_gemm(A, B, path=2)
    assert ei.value.status == 6


def test_repeated_launches_are_consistent(ctx):
    g = torch.Generator(device="cuda").manual_seed(3)
    A = torch.randn(1024, 512, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(2048, 512, device="cuda", generator=g).to(torch.bfloat16)
    C0 = ctx.debug_gemm(A, B, path=2)
    for _ in range(5):
        assert torch.equal(ctx.debug_gemm(A, B, path=2), C0)
