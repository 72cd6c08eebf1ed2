"""The library's GEMMs in isolation: C = A B^T with bf16 operands and fp32
accumulation, on the tcgen05 tensor-core path (one CTA per 128 x 256 tile,
and CTA pairs per 256 x 256 tile) and the CUDA-core path, against torch's
fp32 product of the same bf16 values (ragged M, N and K tails included; for
pairs, M tails that leave the second CTA of a pair partly or wholly past M).
Both operand layouts: K-major (A as M x K rows, B as N x K) and MN-major
(A stored K x M, B stored K x N, as the weight-gradient contraction reads
the error rows and the inputs)."""
import pytest
import torch

import zeroth_order_transformer_dust_b200 as dust

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx(cuda_ok):
    return dust.Context(0)


SHAPES = [(128, 256, 64), (256, 512, 128), (300, 500, 72), (1, 16, 8), (129, 257, 1032),
          (1000, 50304, 64), (2048, 1024, 1024), (4096, 3072, 768), (64, 768, 3072)]


def _check(ctx, M, N, K, path):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N * 3 + K)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    C = ctx.debug_gemm(A, B, path=path)
    ref = A.float() @ B.float().T
    err = ((C - ref).norm() / ref.norm()).item()
    assert err < 1e-5, err


@pytest.mark.parametrize("M,N,K", [(256, 256, 64), (128, 256, 64), (100, 16, 8), (384, 300, 200)])
def test_pair_gemm_small(ctx, M, N, K):
    _check(ctx, M, N, K, 3)


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("path", [2, 1, 3])
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


@pytest.mark.parametrize("path", [2, 3])
def test_repeated_launches_are_consistent(ctx, path):
    g = torch.Generator(device="cuda").manual_seed(3)
    A = torch.randn(1024, 512, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(2048, 512, device="cuda", generator=g).to(torch.bfloat16)
    C0 = ctx.debug_gemm(A, B, path=path)
    for _ in range(5):
        assert torch.equal(ctx.debug_gemm(A, B, path=path), C0)


def test_pair_and_single_cta_paths_agree(ctx):
    g = torch.Generator(device="cuda").manual_seed(5)
    A = torch.randn(1000, 768, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(3000, 768, device="cuda", generator=g).to(torch.bfloat16)
    c2, c3 = ctx.debug_gemm(A, B, path=2), ctx.debug_gemm(A, B, path=3)
    assert ((c2 - c3).norm() / c2.norm()).item() < 1e-6


def test_injected_timeout_is_reported_and_the_context_recovers(ctx):
    # path 4: the tensor-core GEMM with its pipeline waits limited to zero. The
    # kernel gives up, drains its own copies and MMAs, frees TMEM and returns;
    # the call reports DUST_ERR_TIMEOUT and the next call runs normally.
    g = torch.Generator(device="cuda").manual_seed(9)
    A = torch.randn(4096, 4096, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(2048, 4096, device="cuda", generator=g).to(torch.bfloat16)
    with pytest.raises(dust.DustError) as ei:
        ctx.debug_gemm(A, B, path=4)
    assert ei.value.status == 5
    C = ctx.debug_gemm(A, B, path=2)
    ref = A.float() @ B.float().T
    assert ((C - ref).norm() / ref.norm()).item() < 1e-5


MN_SHAPES = [(128, 256, 64), (256, 512, 128), (304, 520, 72), (64, 16, 8), (136, 264, 1032),
             (1000, 1024, 200), (50304, 1024, 256), (1024, 64, 4096), (8, 40, 100)]


def _mn_operands(M, N, K):
    g = torch.Generator(device="cuda").manual_seed(M * 5 + N * 11 + K)
    At = torch.randn(K, M, device="cuda", generator=g).to(torch.bfloat16)
    Bt = torch.randn(K, N, device="cuda", generator=g).to(torch.bfloat16)
    return At, Bt


@pytest.mark.parametrize("M,N,K", MN_SHAPES)
@pytest.mark.parametrize("path", [2, 1, 3, 0])
def test_mn_major_gemm_matches_fp32_product(ctx, M, N, K, path):
    At, Bt = _mn_operands(M, N, K)
    C = ctx.debug_gemm_mn(At, Bt, path=path)
    ref = At.float().T @ Bt.float()
    err = ((C - ref).norm() / ref.norm()).item()
    assert err < 1e-5, err


@pytest.mark.parametrize("path", [2, 3])
@pytest.mark.parametrize("M,N,K", [(304, 520, 72), (1000, 1024, 200), (256, 256, 1032)])
def test_mn_major_equals_k_major_bit_for_bit(ctx, M, N, K, path):
    # the same values in the same k order: the tensor cores give the same sums
    At, Bt = _mn_operands(M, N, K)
    c_mn = ctx.debug_gemm_mn(At, Bt, path=path)
    c_k = ctx.debug_gemm(At.T.contiguous(), Bt.T.contiguous(), path=path)
    assert torch.equal(c_mn, c_k)


def test_mn_major_rows_must_be_16_byte_multiples(ctx):
    At, Bt = _mn_operands(100, 64, 64)           # M = 100: 200-byte rows
    with pytest.raises(dust.DustError) as ei:
        ctx.debug_gemm_mn(At, Bt, path=2)
    assert ei.value.status == 6
    C = ctx.debug_gemm_mn(At, Bt, path=0)        # CUDA cores
    ref = At.float().T @ Bt.float()
    assert ((C - ref).norm() / ref.norm()).item() < 1e-5
