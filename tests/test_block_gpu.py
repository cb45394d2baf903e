"""Block forward/backward parity through the C ABI against the fp64 oracle.

Inputs are the same seeded values on both sides (rounded to the storage
dtype, widened to fp64 for the oracle).  Tolerance: normwise max relative
error <= 2e-2 for bf16 storage, <= 1e-5 for the fp32 configuration."""
import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from helpers import TOL, fp8_mode, judge, np64, oracle_layer, relerr, scalar_err, small_bf16

pytestmark = pytest.mark.gpu


def run_block(gb, c, w, inp, layer):
    from gpt_transformer_block_b200.model import BlockRunner, to_device_weights, zero_grads_like, storage_torch_dtype
    dt = storage_torch_dtype(c)
    dw = to_device_weights(c, w)
    lw = dw["layers"][layer]
    x = inp["x"].to("cuda", dt)
    x0 = inp["x0"].to("cuda", dt)
    dy = inp["dy"].to("cuda", dt)
    idx = inp["idx"].cuda()
    r = BlockRunner(c)
    x_out = torch.empty_like(x)
    r.forward(layer, lw, x, x0, idx, x_out)
    g = zero_grads_like(c, dw)["layers"][layer]
    dx = torch.empty_like(x)
    dx0 = torch.zeros(x.shape, dtype=torch.float32, device="cuda")
    r.backward(layer, lw, x, x0, idx, dy, dx, dx0, g)
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    return x_out, dx, dx0, g


def block_errors(x_out, dx, dx0, g, y, rdx, rdx0, rg):
    """Per-output errors of a block's results against one oracle evaluation."""
    errs = {"x_out": relerr(np64(x_out), y), "dx": relerr(np64(dx), rdx), "dx0": relerr(np64(dx0), rdx0)}
    for k in ("w_qkv", "w_o", "w_fc", "w_proj", "w_ve_gate", "ve_table"):
        if k in rg:
            errs[k] = relerr(np64(g[k]), rg[k])
    lam = np64(g["lambdas"])
    errs["resid_lambda"] = scalar_err(lam[0], rg["resid_lambda"], rg["_scale"]["resid_lambda"])
    errs["x0_lambda"] = scalar_err(lam[1], rg["x0_lambda"], rg["_scale"]["x0_lambda"])
    return errs


def oracle_block(c, lw, inp, layer, f8):
    idx = inp["idx"].numpy()
    y, cache = om.block_forward(c, lw, np64(inp["x"]), np64(inp["x0"]), idx, layer, fp8=f8)
    rdx, rdx0, rg = om.block_backward(c, lw, cache, np64(inp["dy"]), idx, layer, fp8=f8)
    return y, rdx, rdx0, rg


def check_block(gb, c, layer, seed=1, x_std=1.0):
    w = synth.make_weights(c, seed=seed)
    inp = synth.make_block_inputs(c, seed=seed + 1, x_std=x_std)
    x_out, dx, dx0, g = run_block(gb, c, w, inp, layer)
    lw = oracle_layer(w, layer)
    f8 = fp8_mode(c)
    ref = oracle_block(c, lw, inp, layer, f8)
    errs = block_errors(x_out, dx, dx0, g, *ref)
    gpu_exact = ref_exact = None
    if f8:  # the FP8 envelope: distances to the exact (non-FP8) block
        exact = oracle_block(c, lw, inp, layer, False)
        gpu_exact = block_errors(x_out, dx, dx0, g, *exact)
        y, rdx, rdx0, rg = ref
        ref_exact = block_errors(y, rdx, rdx0, {k: v for k, v in rg.items() if k != "_scale"} | {"lambdas": [
            rg["resid_lambda"], rg["x0_lambda"]]}, *exact)
    bad = judge(errs, TOL[c["dtype"]], gpu_exact, ref_exact)
    assert not bad, (bad, errs)
    return errs


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_block_bf16_small(cuda_lib, layer):
    # layer 0: full causal; layer 1: window 48 + value embedding; layer 2: full
    check_block(cuda_lib, small_bf16(), layer)


@pytest.mark.parametrize("layer", [0, 1])
def test_block_bf16_gqa_window(cuda_lib, layer):
    # H=4, Hkv=2 (G=2), H*hd != d, T not a multiple of any tile
    c = small_bf16(n_head=4, n_kv_head=2, T=333, B=1, window=[100, 0, -1], has_ve=[1, 1, 0], n_layer=3)
    check_block(cuda_lib, c, layer)


def test_block_fp32_config(cuda_lib):
    # the fp32 block as specified: B=2, T=64, d=128, H=2, Hkv=1, hd=64, window 32
    c = synth.config("block_fp32")
    check_block(cuda_lib, c, 0)


def test_block_fp32_all_terms(cuda_lib):
    # same block with every term on: value embedding, random lambdas
    c = synth.config("block_fp32", has_ve=[1])
    check_block(cuda_lib, c, 0)


@pytest.mark.parametrize("layer", [0, 1])
@pytest.mark.parametrize("grad", ["e4m3", "e5m2"])
def test_block_fp8(cuda_lib, layer, grad):
    # e4m3 operands with per-tensor scales on the four block GEMMs (fwd, dgrad,
    # wgrad), or e5m2 gradient operands (the variant); the oracle quantises the
    # same bf16 tensors the same way
    c = small_bf16(dtype="fp8", n_layer=2, window=[-1, 48], has_ve=[0, 1], fp8_grad=grad)
    check_block(cuda_lib, c, layer)
