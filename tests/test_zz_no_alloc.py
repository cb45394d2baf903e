"""lm_head_xent_noalloc: the allocation-free variant of lm_head_xent for callers
that cannot allocate device memory (a plugin handed tensors and a stream by a
framework that owns all device memory, or a path that must not call
cudaMalloc); it uses the library's static scratch array instead of a
workspace.  Checked through the C ABI against the existing lm_head_xent on the
same inputs, for two calls in a row (the second call reuses the scratch the
first one left behind), and against the fp64 oracle.  Collected last on
purpose; it also passes on its own in a fresh process."""
import pytest
import torch

from oracle import model as om
from helpers import TOL, np64, relerr, small_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,vocab", [("bf16", 1024), ("bf16", 32768), ("f32", 1024)])
def test_noalloc_matches_lm_head_xent(cuda_lib, dtype, vocab):
    gb = cuda_lib
    from gpt_transformer_block_b200.model import lm_head
    g = torch.Generator().manual_seed(77 + vocab)
    N, d = 300, 256
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    c = small_bf16(B=1, T=N, vocab=vocab, dtype=dtype, head_dim=128 if dtype == "bf16" else 64)
    cfg = gb.make_config(c)
    h_cpu = torch.randn(N, d, generator=g).to(tdt)
    w_cpu = (torch.randn(vocab, d, generator=g) * 0.05).to(tdt)
    y_cpu = torch.randint(0, vocab, (N,), generator=g, dtype=torch.int32)
    h, w, y = h_cpu.cuda(), w_cpu.cuda(), y_cpu.cuda()
    tol = TOL[dtype]

    dh_ref = torch.empty(N, d, dtype=tdt, device="cuda")
    dw_ref = torch.zeros(vocab, d, dtype=torch.float32, device="cuda")
    loss_ref = lm_head(c, h, w, y, dh_ref, dw_ref)
    rl, rdh, rdw = om.lm_head_xent(np64(h_cpu), np64(w_cpu), y_cpu.numpy())

    for _ in range(2):
        dh = torch.full((N, d), float("nan"), dtype=tdt, device="cuda")
        dw = torch.zeros(vocab, d, dtype=torch.float32, device="cuda")
        loss = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
        gb.lm_head_xent_noalloc(cfg, h, w, y, loss, dh, dw)
        torch.cuda.synchronize()
        assert gb.gptb_device_error() == 0
        assert abs(loss.item() - loss_ref.item()) <= tol * abs(loss_ref.item())
        assert relerr(np64(dh), np64(dh_ref)) <= tol
        assert relerr(np64(dw), np64(dw_ref)) <= tol
        assert abs(loss.item() - rl) <= tol * abs(rl)
        assert relerr(np64(dh), rdh) <= tol
        assert relerr(np64(dw), rdw) <= tol


def test_noalloc_rejects_too_many_rows(cuda_lib):
    gb = cuda_lib
    c = small_bf16(B=2, T=40000, vocab=1024)
    cfg = gb.make_config(c)
    t = torch.zeros(8, dtype=torch.float32, device="cuda")
    with pytest.raises(gb.GPTBError) as e:
        gb.lm_head_xent_noalloc(cfg, t, t, t, t, t, t)
    assert e.value.code == gb.ERR_WORKSPACE
