"""Full-size parity at the configurations' widths and sequence length (T=2048).

1. One block at full width (B=1, or B=2 for FP8 so that the per-tensor scales
   see more than one batch row), forward and backward through the C ABI,
   against the fp64 oracle: the block output, dx, dx0 and EVERY gradient
   (w_qkv, w_o, w_fc, w_proj, w_ve_gate, ve_table and both lambdas).  Both
   window kinds of d20_gqa (window 1024 on even layers, full on odd ones) are
   covered, and value-embedding layers of every config.
2. The benchmark's launch configuration (B=16, T=2048): sampled batch rows
   of the block output, dx and dx0 checked against the oracle run on those
   rows alone (rows are independent in the forward and in dx / dx0; bf16
   only, since FP8's per-tensor scales depend on every row)."""
import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from helpers import TOL, fp8_mode, judge, np64, oracle_layer, relerr

pytestmark = pytest.mark.gpu


def _run_block(c, w, inp, layer):
    from gpt_transformer_block_b200.model import BlockRunner, to_device_weights, zero_grads_like
    dw = to_device_weights(c, w)
    lw = dw["layers"][layer]
    x = inp["x"].to("cuda", torch.bfloat16)
    x0 = inp["x0"].to("cuda", torch.bfloat16)
    dy = inp["dy"].to("cuda", torch.bfloat16)
    idx = inp["idx"].cuda()
    r = BlockRunner(c)
    x_out = torch.empty_like(x)
    r.forward(layer, lw, x, x0, idx, x_out)
    g = zero_grads_like(c, dw)["layers"][layer]
    dx = torch.empty_like(x)
    dx0 = torch.zeros(x.shape, dtype=torch.float32, device="cuda")
    r.backward(layer, lw, x, x0, idx, dy, dx, dx0, g)
    torch.cuda.synchronize()
    return x_out, dx, dx0, g


@pytest.mark.parametrize("name,layer,B", [("d12", 11, 1), ("d12", 10, 1), ("d20_gqa", 18, 1), ("d20_gqa", 19, 1),
                                          ("d24", 23, 1), ("d24", 12, 1), ("d26_fp8", 25, 2), ("d26_fp8", 0, 2)])
def test_block_full_width_every_gradient(cuda_lib, name, layer, B):
    c = synth.config(name, B=B)
    w = synth.make_weights(c, seed=201 + layer)
    inp = synth.make_block_inputs(c, seed=202 + layer)
    x_out, dx, dx0, g = _run_block(c, w, inp, layer)
    assert cuda_lib.gptb_device_error() == 0
    from test_block_gpu import block_errors, oracle_block
    lw = oracle_layer(w, layer)
    f8 = fp8_mode(c)
    ref = oracle_block(c, lw, inp, layer, f8)
    errs = block_errors(x_out, dx, dx0, g, *ref)
    assert ("ve_table" in errs) == bool(c["has_ve"][layer])
    gpu_exact = ref_exact = None
    if f8:  # the FP8 envelope (tests/helpers.py): distances to the exact block
        exact = oracle_block(c, lw, inp, layer, False)
        gpu_exact = block_errors(x_out, dx, dx0, g, *exact)
        y, rdx, rdx0, rg = ref
        ref_exact = block_errors(y, rdx, rdx0, {k: v for k, v in rg.items() if k != "_scale"} | {"lambdas": [
            rg["resid_lambda"], rg["x0_lambda"]]}, *exact)
    bad = judge(errs, TOL[c["dtype"]], gpu_exact, ref_exact)
    assert not bad, (bad, errs)


@pytest.mark.parametrize("name,layer,rows", [("d24", 23, (0, 15)), ("d20_gqa", 0, (7,)), ("d12", 11, (3,))])
def test_block_bench_shape_sampled_rows(cuda_lib, name, layer, rows):
    c = synth.config(name)
    w = synth.make_weights(c, seed=101)
    inp = synth.make_block_inputs(c, seed=102)
    x_out, dx, dx0, _ = _run_block(c, w, inp, layer)
    assert cuda_lib.gptb_device_error() == 0
    olw = oracle_layer(w, layer)
    tol = TOL[c["dtype"]]
    for b in rows:
        c1 = dict(c, B=1)
        sl = slice(b, b + 1)
        y, cache = om.block_forward(c1, olw, np64(inp["x"][sl]), np64(inp["x0"][sl]), inp["idx"][sl].numpy(), layer)
        rdx, rdx0, _ = om.block_backward(c1, olw, cache, np64(inp["dy"][sl]), inp["idx"][sl].numpy(), layer)
        errs = {"x_out": relerr(np64(x_out[sl]), y), "dx": relerr(np64(dx[sl]), rdx),
                "dx0": relerr(np64(dx0[sl]), rdx0)}
        assert all(v <= tol for v in errs.values()), (b, errs)
