"""Failure detection on the GPU without a fault: a CTA waits on an mbarrier
that nothing ever arrives on.  The bounded wait must expire, the kernel must
record it and return, the host must read GPTB_ERR_TIMEOUT, and the context
must stay usable for the next launch."""
import pytest
import torch

from helpers import relerr

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_survives(cuda_lib):
    gb = cuda_lib
    assert gb.gptb_device_error() == 0
    assert gb.gptb_probe_bounded_wait(2_000_000) == gb.ERR_TIMEOUT   # 2 ms limit
    assert gb.gptb_device_error() == 0                               # error word was cleared
    # the context still runs the tensor-core GEMM correctly afterwards
    g = torch.Generator().manual_seed(1)
    A = (torch.randn(256, 128, generator=g) * 0.5).to(torch.bfloat16)
    B = (torch.randn(264, 128, generator=g) * 0.5).to(torch.bfloat16)
    C = torch.zeros(256, 264, dtype=torch.float32, device="cuda")
    gb.gptb_gemm_bf16(A.cuda(), 0, 128, B.cuda(), 0, 128, C, 1, 264, 256, 264, 128)
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    assert relerr(C.cpu().double().numpy(), A.double().numpy() @ B.double().numpy().T) < 1e-5
