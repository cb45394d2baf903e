"""Decode attention over a KV cache through the C ABI against the fp64 oracle
(oracle/decode.py): GQA and MHA, full and windowed, ragged lengths including 1
and the full cache, the d24 shape, the largest supported group (8 query heads
per kv head; more are rejected), more key pieces than the persistent grid has
CTAs, and a sequence whose length is outside the cache (o = 0, lse = -inf)."""
import numpy as np
import pytest
import torch

from helpers import TOL, relerr
from oracle import decode as od

pytestmark = pytest.mark.gpu


def _run(gb, B, H, Hk, Tmax, lens, window, seed=0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, 128, generator=g).bfloat16()
    k = torch.randn(B, Tmax, Hk, 128, generator=g).bfloat16()
    v = torch.randn(B, Tmax, Hk, 128, generator=g).bfloat16()
    ln = torch.tensor(lens, dtype=torch.int32)
    o = torch.empty(B, H, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(gb.gptb_decode_workspace_bytes(B, H, Tmax), dtype=torch.uint8, device="cuda")
    gb.gptb_decode_attention(q.cuda(), k.cuda(), v.cuda(), ln.cuda(), o, lse, B, H, Hk, Tmax, window, ws)
    torch.cuda.synchronize()
    return q, k, v, ln, o.cpu(), lse.cpu()


@pytest.mark.parametrize("window", [-1, 0, 37])
def test_decode_gqa_ragged(cuda_lib, window):
    B, H, Hk, Tmax = 6, 4, 2, 600
    lens = [600, 1, 129, 64, 257, 513]  # several key pieces of 128, ragged last pieces
    q, k, v, ln, o, lse = _run(cuda_lib, B, H, Hk, Tmax, lens, window)
    ro, rl = od.decode_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), lens, window)
    assert relerr(o.double().numpy(), ro) <= TOL["bf16"]
    assert np.max(np.abs(lse.double().numpy() - rl)) <= 1e-4 * max(1.0, np.max(np.abs(rl)))


def test_decode_d24_shape(cuda_lib):
    B, H, Hk, Tmax = 4, 12, 12, 2048
    lens = [2048, 1500, 700, 2]
    q, k, v, ln, o, lse = _run(cuda_lib, B, H, Hk, Tmax, lens, -1, seed=1)
    ro, rl = od.decode_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), lens, -1)
    assert relerr(o.double().numpy(), ro) <= TOL["bf16"]
    assert np.max(np.abs(lse.double().numpy() - rl)) <= 1e-4 * max(1.0, np.max(np.abs(rl)))


def test_decode_length_outside_cache(cuda_lib):
    B, H, Hk, Tmax = 3, 2, 1, 64
    lens = [10, 0, 65]
    q, k, v, ln, o, lse = _run(cuda_lib, B, H, Hk, Tmax, lens, -1, seed=2)
    ro, rl = od.decode_attention(q[:1].double().numpy(), k[:1].double().numpy(), v[:1].double().numpy(), lens[:1], -1)
    assert relerr(o[:1].double().numpy(), ro) <= TOL["bf16"]
    assert torch.all(o[1:] == 0)
    assert torch.all(torch.isinf(lse[1:])) and torch.all(lse[1:] < 0)


@pytest.mark.parametrize("window", [-1, 200])
def test_decode_group_of_eight(cuda_lib, window):
    B, H, Hk, Tmax = 3, 16, 2, 700
    lens = [700, 130, 5]
    q, k, v, ln, o, lse = _run(cuda_lib, B, H, Hk, Tmax, lens, window, seed=3)
    ro, rl = od.decode_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), lens, window)
    assert relerr(o.double().numpy(), ro) <= TOL["bf16"]
    assert np.max(np.abs(lse.double().numpy() - rl)) <= 1e-4 * max(1.0, np.max(np.abs(rl)))


def test_decode_group_of_nine_rejected(cuda_lib):
    gb = cuda_lib
    B, H, Hk, Tmax = 1, 9, 1, 64
    t = torch.zeros(B * Tmax * H * 128, dtype=torch.bfloat16, device="cuda")
    ln = torch.tensor([10], dtype=torch.int32, device="cuda")
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(gb.gptb_decode_workspace_bytes(B, H, Tmax), dtype=torch.uint8, device="cuda")
    with pytest.raises(gb.GPTBError) as e:
        gb.gptb_decode_attention(t, t, t, ln, t, lse, B, H, Hk, Tmax, -1, ws)
    assert e.value.code == gb.ERR_UNSUPPORTED


def test_decode_many_pieces_per_cta(cuda_lib):
    """48 sequences x 2 kv heads x 16 pieces: several pieces per persistent CTA,
    so the stage ring wraps many times and both consumer groups alternate."""
    B, H, Hk, Tmax = 48, 4, 2, 2048
    g = torch.Generator().manual_seed(9)
    lens = torch.randint(1, Tmax + 1, (B,), generator=g).tolist()
    q, k, v, ln, o, lse = _run(cuda_lib, B, H, Hk, Tmax, lens, -1, seed=4)
    ro, rl = od.decode_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), lens, -1)
    assert relerr(o.double().numpy(), ro) <= TOL["bf16"]
    assert np.max(np.abs(lse.double().numpy() - rl)) <= 1e-4 * max(1.0, np.max(np.abs(rl)))
