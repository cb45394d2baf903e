"""tcgen05 GEMM parity (all three operand layouts, ragged tiles, split-K
accumulation) against an fp64 matmul of the same bf16 operands."""
import numpy as np
import pytest
import torch

from helpers import relerr

pytestmark = pytest.mark.gpu


def _mk(shape, g):
    return (torch.randn(*shape, generator=g) * 0.5).to(torch.bfloat16)


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 1), (1, 0)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (296, 264, 200), (1000, 520, 1536), (8, 8, 8)])
def test_gemm_layouts(cuda_lib, a_mn, b_mn, M, N, K):
    gb = cuda_lib
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    A = _mk((M, K), g)
    B = _mk((N, K), g)
    ref = A.double().numpy() @ B.double().numpy().T
    As = (A.t().contiguous() if a_mn else A).cuda()
    Bs = (B.t().contiguous() if b_mn else B).cuda()
    lda = M if a_mn else K
    ldb = N if b_mn else K
    # fp32 accumulate (+=) twice -> 2 * A B^T
    C = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    gb.gptb_gemm_bf16(As, a_mn, lda, Bs, b_mn, ldb, C, 1, N, M, N, K)
    gb.gptb_gemm_bf16(As, a_mn, lda, Bs, b_mn, ldb, C, 1, N, M, N, K)
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    assert relerr(C.cpu().double().numpy(), 2 * ref) < 1e-5
    # bf16 store
    Cb = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    gb.gptb_gemm_bf16(As, a_mn, lda, Bs, b_mn, ldb, Cb, 0, N, M, N, K)
    torch.cuda.synchronize()
    assert relerr(Cb.float().cpu().numpy(), ref) < 8e-3


def test_gemm_long_k_split(cuda_lib):
    """Weight-gradient shape: few tiles, long K -> split-K partial sums meet in fp32."""
    gb = cuda_lib
    g = torch.Generator().manual_seed(5)
    M, N, K = 256, 512, 32768
    A = _mk((K, M), g)   # stored [K, M]: M-major
    B = _mk((K, N), g)   # stored [K, N]: N-major
    ref = A.double().numpy().T @ B.double().numpy()
    C = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    gb.gptb_gemm_bf16(A.cuda(), 1, M, B.cuda(), 1, N, C, 1, N, M, N, K)
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    assert relerr(C.cpu().double().numpy(), ref) < 1e-5


def test_gemm_rejects_misaligned(cuda_lib):
    gb = cuda_lib
    A = torch.zeros(64, 100, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(64, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(gb.GPTBError):
        gb.gptb_gemm_bf16(A, 0, 100 - 1, A, 0, 100, C, 1, 64, 64, 64, 96)


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (304, 272, 208), (1008, 528, 1536)])
@pytest.mark.parametrize("e5m2", [False, True])
def test_gemm_fp8_matches_oracle_product(cuda_lib, a_mn, b_mn, M, N, K, e5m2):
    """The FP8 tensor-core GEMM (single-CTA and CTA-pair forms, every layout
    the block uses, e4m3 or e5m2 A) against the oracle's quantised product of
    the same bf16 operands: identical codes, so only the fp32 accumulation
    order differs."""
    from oracle import fp8 as of
    gb = cuda_lib
    g = torch.Generator().manual_seed(M + N + K + (7 if e5m2 else 0))
    A = _mk((M, K), g)
    B = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    a, b = A.double().numpy(), B.double().numpy()
    ref = of.fp8_matmul_grad(a, b.T) if e5m2 else of.fp8_matmul(a, b.T)
    As = (A.t().contiguous() if a_mn else A).cuda()
    Bs = (B.t().contiguous() if b_mn else B).cuda()
    C = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    gb.gptb_gemm_fp8(As, a_mn, M if a_mn else K, Bs, b_mn, N if b_mn else K, C, N, M, N, K, e5m2)
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    assert relerr(C.cpu().double().numpy(), ref) < 1e-5


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("M,N,K,batch", [(128, 256, 64, 3), (304, 264, 200, 2), (768, 768, 768, 5)])
def test_gemm_batched(cuda_lib, a_mn, b_mn, M, N, K, batch):
    """One launch over `batch` matrices stored one after another (the batch
    entry is the third coordinate of the tensor maps): each product against an
    fp64 matmul, for a bf16 store and an fp32 accumulation (split-K may meet
    the batch), in the single-CTA (M < 256) and CTA-pair forms."""
    gb = cuda_lib
    g = torch.Generator().manual_seed(M + N + K + batch)
    A = [_mk((M, K), g) for _ in range(batch)]
    B = [_mk((N, K), g) for _ in range(batch)]
    As = torch.stack([a.t().contiguous() if a_mn else a for a in A]).cuda()
    Bs = torch.stack([b.t().contiguous() if b_mn else b for b in B]).cuda()
    lda = M if a_mn else K
    ldb = N if b_mn else K
    C = torch.zeros(batch, M, N, dtype=torch.float32, device="cuda")
    gb.gptb_gemm_bf16_batched(As, a_mn, lda, M * K, Bs, b_mn, ldb, N * K, C, 1, N, M * N, M, N, K, batch)
    Cb = torch.empty(batch, M, N, dtype=torch.bfloat16, device="cuda")
    gb.gptb_gemm_bf16_batched(As, a_mn, lda, M * K, Bs, b_mn, ldb, N * K, Cb, 0, N, M * N, M, N, K, batch)
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    for i in range(batch):
        ref = A[i].double().numpy() @ B[i].double().numpy().T
        assert relerr(C[i].cpu().double().numpy(), ref) < 1e-5, i
        assert relerr(Cb[i].float().cpu().numpy(), ref) < 8e-3, i
