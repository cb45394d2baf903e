"""lm_head_xent and gpt_stack_step parity through the C ABI against the
fp64 oracle (loss and every gradient)."""
import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from helpers import TOL, fp8_mode, judge, np64, oracle_weights, relerr, scalar_err, small_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,N,V", [("bf16", 300, 1024), ("f32", 300, 1024), ("bf16", 300, 1000),
                                       ("bf16", 9192, 32768)])
def test_lm_head_xent(cuda_lib, dtype, N, V):
    """N=9192 at the vocabulary of every stack config: two row chunks (8192 +
    a ragged 1000), dW_lm accumulated across them; V=1000 leaves the last
    256-column tile of the logits GEMM partly outside the vocabulary."""
    from gpt_transformer_block_b200.model import lm_head
    g = torch.Generator().manual_seed(3)
    d = 256
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    h = torch.randn(N, d, generator=g).to(tdt)
    w = (torch.randn(V, d, generator=g) * 0.05).to(tdt)
    y = torch.randint(0, V, (N,), generator=g, dtype=torch.int32)
    c = small_bf16(B=1, T=N, vocab=V, dtype=dtype, head_dim=128 if dtype == "bf16" else 64)
    dh = torch.empty(N, d, dtype=tdt, device="cuda")
    dw = torch.zeros(V, d, dtype=torch.float32, device="cuda")
    loss = lm_head(c, h.cuda(), w.cuda(), y.cuda(), dh, dw)
    torch.cuda.synchronize()
    assert cuda_lib.gptb_device_error() == 0
    rl, rdh, rdw = om.lm_head_xent(np64(h), np64(w), y.numpy())
    tol = TOL[dtype]
    assert abs(loss.item() - rl) / abs(rl) <= tol
    assert relerr(np64(dh), rdh) <= tol
    assert relerr(np64(dw), rdw) <= tol


def run_stack(gb, c, w, batch):
    from gpt_transformer_block_b200.model import GPTStack
    st = GPTStack(c, w)
    loss = st.step(batch["idx"].cuda(), batch["targets"].cuda())
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    return loss.item(), st.g


def stack_errors(loss, g, rl, rg, top, layers):
    """Per-output errors of a stack step's results against one oracle evaluation."""
    errs = {"loss": abs(loss - rl) / abs(rl)}
    for k in ("wte", "w_lm", "w_smear_gate"):
        if k in rg and k in top:
            errs[k] = relerr(np64(g[k]), rg[k])
    for k in ("smear_lambda", "backout_lambda"):
        if k in rg and k in top:
            errs[k] = scalar_err(np64(g[k])[0], rg[k], rg["_scale"][k])
    for i, lg in enumerate(rg["layers"]):
        if layers is not None and i not in layers:
            continue
        lam = np64(g["layers"][i]["lambdas"])
        for k, v in lg.items():
            if k == "_scale":
                continue
            if k in ("resid_lambda", "x0_lambda"):
                errs[f"L{i}.{k}"] = scalar_err(lam[0 if k == "resid_lambda" else 1], v, lg["_scale"][k])
            else:
                errs[f"L{i}.{k}"] = relerr(np64(g["layers"][i][k]), v)
    return errs


def _as_grads(rg):
    """An oracle gradient tree in the layout of the GPU's (lambdas as pairs)."""
    g = {k: (np.array([v]) if isinstance(v, float) else v) for k, v in rg.items() if k not in ("layers", "_scale")}
    g["layers"] = [dict({k: v for k, v in lg.items() if k not in ("_scale", "resid_lambda", "x0_lambda")},
                        lambdas=np.array([lg["resid_lambda"], lg["x0_lambda"]])) for lg in rg["layers"]]
    return g


def compare_stack(c, w, batch, loss, g, layers=None, top=("wte", "w_lm", "w_smear_gate", "smear_lambda",
                                                          "backout_lambda")):
    ow = oracle_weights(w)
    f8 = fp8_mode(c)
    idx, tg = batch["idx"].numpy(), batch["targets"].numpy()
    rl, cache = om.stack_forward(c, ow, idx, tg, fp8=f8)
    rg = om.stack_backward(c, ow, cache, idx, fp8=f8)
    errs = stack_errors(loss, g, rl, rg, top, layers)
    gpu_exact = ref_exact = None
    if f8:  # the FP8 envelope: distances to the exact (non-FP8) stack
        c0 = dict(c, fp8_lm_head=False)
        rl0, cache0 = om.stack_forward(c0, ow, idx, tg, fp8=False)
        rg0 = om.stack_backward(c0, ow, cache0, idx, fp8=False)
        gpu_exact = stack_errors(loss, g, rl0, rg0, top, layers)
        ref_exact = stack_errors(rl, _as_grads(rg), rl0, rg0, top, layers)
    bad = judge(errs, TOL[c["dtype"]], gpu_exact, ref_exact)
    assert not bad, (bad, errs)
    return errs


def test_stack_bf16_small(cuda_lib):
    c = small_bf16()
    w = synth.make_weights(c, seed=11)
    b = synth.make_batch(c, seed=12)
    loss, g = run_stack(cuda_lib, c, w, b)
    compare_stack(c, w, b, loss, g)


def test_stack_bf16_gqa_backout0(cuda_lib):
    c = small_bf16(n_head=4, n_kv_head=2, n_layer=2, window=[64, -1], has_ve=[1, 0], backout_layer=0, T=130)
    w = synth.make_weights(c, seed=21)
    b = synth.make_batch(c, seed=22)
    loss, g = run_stack(cuda_lib, c, w, b)
    compare_stack(c, w, b, loss, g)


def test_stack_fp32_all_terms(cuda_lib):
    # the fp32 block width/heads at stack level with VE, smear, backout on
    c = synth.config("block_fp32", n_layer=2, has_ve=[0, 1], smear_ch=24, backout_layer=1, lm_head=True,
                     vocab=512, window=[32, -1])
    w = synth.make_weights(c, seed=31)
    b = synth.make_batch(c, seed=32)
    loss, g = run_stack(cuda_lib, c, w, b)
    compare_stack(c, w, b, loss, g)


def test_grad_accumulation_equals_sum(cuda_lib):
    """Two steps without zeroing accumulate exactly twice one step's gradients
    (the property gradient accumulation relies on)."""
    from gpt_transformer_block_b200.model import GPTStack
    c = small_bf16(n_layer=2, window=[-1, 32], has_ve=[0, 1])
    w = synth.make_weights(c, seed=41)
    b = synth.make_batch(c, seed=42)
    st = GPTStack(c, w)
    idx, tg = b["idx"].cuda(), b["targets"].cuda()
    st.step(idx, tg)
    one = st.g["layers"][1]["w_qkv"].clone()
    st.step(idx, tg)
    torch.cuda.synchronize()
    two = st.g["layers"][1]["w_qkv"]
    assert relerr(two.cpu().numpy(), 2 * one.cpu().numpy()) < 1e-5


def test_stack_fp8_small(cuda_lib):
    """FP8 end to end (every GEMM product of every block in e4m3): the loss and
    every gradient of every layer, the embedding and the smear / backout terms."""
    c = small_bf16(dtype="fp8")
    w = synth.make_weights(c, seed=51)
    b = synth.make_batch(c, seed=52)
    loss, g = run_stack(cuda_lib, c, w, b)
    compare_stack(c, w, b, loss, g)


def test_stack_fp8_variant_small(cuda_lib):
    """The FP8 variant end to end: e5m2 gradient operands in every block's
    backward GEMMs and the lm_head in FP8 (e4m3 logits, FP8 logits gradient
    with its fixed scale): the loss and every gradient of every layer."""
    c = small_bf16(dtype="fp8", fp8_grad="e5m2", fp8_lm_head=True)
    w = synth.make_weights(c, seed=53)
    b = synth.make_batch(c, seed=54)
    loss, g = run_stack(cuda_lib, c, w, b)
    compare_stack(c, w, b, loss, g)


@pytest.mark.parametrize("grad", ["e4m3", "e5m2"])
def test_lm_head_fp8(cuda_lib, grad):
    """FP8 lm_head at the stack configs' vocabulary over two row chunks (8192 +
    a ragged 1000): e4m3 hf and W_lm, the logits gradient with the fixed scale
    of its 1/N bound in e4m3 or e5m2; against the oracle's FP8 lm_head."""
    from gpt_transformer_block_b200.model import lm_head
    g = torch.Generator().manual_seed(13)
    N, d, V = 9192, 256, 32768
    h = torch.randn(N, d, generator=g).to(torch.bfloat16)
    w = (torch.randn(V, d, generator=g) * 0.05).to(torch.bfloat16)
    y = torch.randint(0, V, (N,), generator=g, dtype=torch.int32)
    c = small_bf16(B=1, T=N, vocab=V, dtype="fp8", fp8_grad=grad, fp8_lm_head=True)
    dh = torch.empty(N, d, dtype=torch.bfloat16, device="cuda")
    dw = torch.zeros(V, d, dtype=torch.float32, device="cuda")
    loss = lm_head(c, h.cuda(), w.cuda(), y.cuda(), dh, dw)
    torch.cuda.synchronize()
    assert cuda_lib.gptb_device_error() == 0
    rl, rdh, rdw = om.lm_head_xent(np64(h), np64(w), y.numpy(), fp8=fp8_mode(c))
    l0, dh0, dw0 = om.lm_head_xent(np64(h), np64(w), y.numpy())
    errs = {"loss": abs(loss.item() - rl) / abs(rl), "dh": relerr(np64(dh), rdh), "dw": relerr(np64(dw), rdw)}
    gpu_exact = {"loss": abs(loss.item() - l0) / abs(l0), "dh": relerr(np64(dh), dh0), "dw": relerr(np64(dw), dw0)}
    ref_exact = {"loss": abs(rl - l0) / abs(l0), "dh": relerr(rdh, dh0), "dw": relerr(rdw, dw0)}
    bad = judge(errs, TOL["fp8"], gpu_exact, ref_exact)
    assert not bad, (bad, errs)


def test_lm_head_out_of_range_targets_are_reported(cuda_lib):
    """Targets -1 and V are never used as indices: the call completes, the
    device error check reports GPTB_ERR_BAD_INPUT, and the other rows' loss
    terms are unchanged (the bad rows add 0 to the mean)."""
    from gpt_transformer_block_b200.model import lm_head
    g = torch.Generator().manual_seed(9)
    N, d, V = 64, 256, 1024
    for dtype in ("bf16", "f32"):
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        h = torch.randn(N, d, generator=g).to(tdt)
        w = (torch.randn(V, d, generator=g) * 0.05).to(tdt)
        y = torch.randint(0, V, (N,), generator=g, dtype=torch.int32)
        y[5], y[40] = -1, V
        c = small_bf16(B=1, T=N, vocab=V, dtype=dtype, head_dim=128 if dtype == "bf16" else 64)
        dh = torch.empty(N, d, dtype=tdt, device="cuda")
        dw = torch.zeros(V, d, dtype=torch.float32, device="cuda")
        loss = lm_head(c, h.cuda(), w.cuda(), y.cuda(), dh, dw)
        assert cuda_lib.gptb_device_error() == cuda_lib.ERR_BAD_INPUT
        assert cuda_lib.gptb_device_error() == 0  # the error word was cleared
        keep = np.ones(N, dtype=bool)
        keep[[5, 40]] = False
        rl, _, _ = om.lm_head_xent(np64(h)[keep], np64(w), y.numpy()[keep])
        assert abs(loss.item() - rl * keep.sum() / N) <= TOL[dtype] * abs(rl)
