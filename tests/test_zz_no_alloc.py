"""lm_head_xent_noalloc: the allocation-free variant of lm_head_xent for callers
that cannot allocate device memory (it uses the library's static scratch
array instead of a workspace).  Checked through the C ABI against the
existing lm_head_xent on the same inputs, for two calls in a row (the second
call reuses the scratch the first one left behind).  Collected last on
purpose; it also passes on its own in a fresh process."""
import pytest
import torch

from helpers import TOL, np64, relerr, small_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("vocab", [1024, 32768])
def test_noalloc_matches_lm_head_xent(cuda_lib, vocab):
    gb = cuda_lib
    from gpt_transformer_block_b200.model import lm_head
    g = torch.Generator().manual_seed(77 + vocab)
    N, d = 300, 256
    c = small_bf16(B=1, T=N, vocab=vocab)
    cfg = gb.make_config(c)
    h = torch.randn(N, d, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(vocab, d, generator=g) * 0.05).to(torch.bfloat16).cuda()
    y = torch.randint(0, vocab, (N,), generator=g, dtype=torch.int32).cuda()

    dh_ref = torch.empty(N, d, dtype=torch.bfloat16, device="cuda")
    dw_ref = torch.zeros(vocab, d, dtype=torch.float32, device="cuda")
    loss_ref = lm_head(c, h, w, y, dh_ref, dw_ref)

    for _ in range(2):
        dh = torch.full((N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        dw = torch.zeros(vocab, d, dtype=torch.float32, device="cuda")
        loss = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
        gb.lm_head_xent_noalloc(cfg, h, w, y, loss, dh, dw)
        torch.cuda.synchronize()
        assert gb.gptb_device_error() == 0
        assert abs(loss.item() - loss_ref.item()) <= TOL["bf16"] * abs(loss_ref.item())
        assert relerr(np64(dh), np64(dh_ref)) <= TOL["bf16"]
        assert relerr(np64(dw), np64(dw_ref)) <= TOL["bf16"]


def test_noalloc_rejects_too_many_rows(cuda_lib):
    gb = cuda_lib
    c = small_bf16(B=2, T=40000, vocab=1024)
    cfg = gb.make_config(c)
    t = torch.zeros(8, dtype=torch.float32, device="cuda")
    with pytest.raises(gb.GPTBError) as e:
        gb.lm_head_xent_noalloc(cfg, t, t, t, t, t, t)
    assert e.value.code == gb.ERR_WORKSPACE
