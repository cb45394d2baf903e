"""Pins of the decode-attention oracle (oracle/decode.py), CPU only: it must
equal the training-time attention's row of the newest token (the prefill of
the same prefix), torch's scaled_dot_product_attention on the single query
with the visibility mask spelled out, and o = v of the newest token when the
window is 0."""
import numpy as np
import pytest
import torch

from oracle import decode as od
from oracle import model as om


def _case(seed, B=3, H=4, Hk=2, hd=16, Tmax=40):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, hd))
    k = rng.standard_normal((B, Tmax, Hk, hd))
    v = rng.standard_normal((B, Tmax, Hk, hd))
    lens = np.array([Tmax, 17, 1][:B])
    return q, k, v, lens


@pytest.mark.parametrize("window", [-1, 5, 0, 100])
def test_decode_equals_last_prefill_row(window):
    q, k, v, lens = _case(1)
    o, lse = od.decode_attention(q, k, v, lens, window)
    for b, L in enumerate(lens):
        # prefill of the prefix 0..L-1 with the decode query in the last row
        qf = np.zeros((1, L, q.shape[1], q.shape[2]))
        qf[0, L - 1] = q[b]
        of, lf = om.attention_forward(qf, k[b:b + 1, :L], v[b:b + 1, :L], window)
        assert np.allclose(o[b], of[0, L - 1], atol=1e-12)
        assert np.allclose(lse[b], lf[0, :, L - 1], atol=1e-12)


def test_decode_matches_torch_sdpa():
    q, k, v, lens = _case(2)
    W = 7
    o, _ = od.decode_attention(q, k, v, lens, W)
    G = q.shape[1] // k.shape[2]
    for b, L in enumerate(lens):
        kk = torch.tensor(k[b, :L]).repeat_interleave(G, dim=1).transpose(0, 1)  # [H, L, hd]
        vv = torch.tensor(v[b, :L]).repeat_interleave(G, dim=1).transpose(0, 1)
        qq = torch.tensor(q[b])[:, None, :]                                        # [H, 1, hd]
        pos = torch.arange(L)
        mask = (pos <= L - 1) & (pos >= L - 1 - W)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask[None, None, :])
        assert np.allclose(o[b], ref[:, 0, :].numpy(), atol=1e-12)


def test_window_zero_returns_the_newest_value():
    q, k, v, lens = _case(3)
    o, _ = od.decode_attention(q, k, v, lens, 0)
    G = q.shape[1] // k.shape[2]
    for b, L in enumerate(lens):
        for h in range(q.shape[1]):
            assert np.allclose(o[b, h], v[b, L - 1, h // G], atol=1e-14)
