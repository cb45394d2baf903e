"""Seeded synthetic inputs and workload presets for the GPT block stack.

This module is shared by the tests, the benchmark and the smoke check. It holds
no arithmetic of the method itself: it only draws random numbers (torch CPU
generator, fixed seeds), rounds them to the storage dtype and names the
workload shapes.  Both the fp64 oracle and the CUDA path consume what it
returns; neither is imported here.

Workloads follow the nanochat GPT model described on the source pages
("How nanochat works / 1. The GPT model": RoPE, QK normalisation, untied
embeddings, ReLU^2 MLP, GQA, sliding windows, value embeddings on alternating
layers, per-layer residual lambdas, smear and backout), at the five sizes the
benchmark and parity suite use.  The pages train on web text (ClimbMix /
FineWeb-EDU); uniform random token ids stand in for it here.
"""
from __future__ import annotations

import copy
import numpy as np
import torch

VOCAB = 32768

# ---------------------------------------------------------------------------
# Workload presets.  Every field is plain data.
#   window[i]  : -1 = full causal, else W (keys j with t-W <= j <= t visible)
#   has_ve[i]  : 1 if layer i adds a gated value embedding
#   backout_layer : index of the layer whose INPUT is saved and subtracted
#                   (scaled) after the last layer; -1 = off
#   smear_ch   : channels feeding the smear gate (0 = smear off)
# ---------------------------------------------------------------------------


def _alternating_ve(n_layer: int) -> list[int]:
    # value embeddings on every other layer, the last layer included
    return [1 if (i % 2) == ((n_layer - 1) % 2) else 0 for i in range(n_layer)]


def _stack(name, n_layer, d, n_head, n_kv_head, window, dtype="bf16", B=16, T=2048):
    return dict(
        name=name, B=B, T=T, d=d, n_head=n_head, n_kv_head=n_kv_head,
        head_dim=128, mlp_hidden=4 * d, vocab=VOCAB, n_layer=n_layer,
        window=list(window), has_ve=_alternating_ve(n_layer),
        ve_gate_ch=32, smear_ch=24, backout_layer=n_layer // 2,
        rope_base=10000.0, norm_eps=1e-6, dtype=dtype, lm_head=True,
    )


CONFIGS = {
    # one block, fp32, small: the oracle finishes it in milliseconds
    "block_fp32": dict(
        name="block_fp32", B=2, T=64, d=128, n_head=2, n_kv_head=1, head_dim=64,
        mlp_hidden=512, vocab=VOCAB, n_layer=1, window=[32], has_ve=[0],
        ve_gate_ch=32, smear_ch=0, backout_layer=-1, rope_base=10000.0,
        norm_eps=1e-6, dtype="f32", lm_head=False,
    ),
    "d12": _stack("d12", 12, 768, 6, 6, [-1] * 12),
    "d20_gqa": _stack("d20_gqa", 20, 1280, 10, 5,
                      [1024 if i % 2 == 0 else -1 for i in range(20)]),
    "d24": _stack("d24", 24, 1536, 12, 12, [-1] * 24),
    "d26_fp8": _stack("d26_fp8", 26, 1664, 13, 13, [-1] * 26, dtype="fp8"),
    # the d26 shape in bf16: the reference point for the FP8 configuration's step time
    "d26_bf16": _stack("d26_bf16", 26, 1664, 13, 13, [-1] * 26),
    # the FP8 variant of the next rows: e5m2 gradient operands and an FP8 lm_head
    "d26_fp8_e5m2": dict(_stack("d26_fp8_e5m2", 26, 1664, 13, 13, [-1] * 26, dtype="fp8"),
                         fp8_grad="e5m2", fp8_lm_head=True),
}

CONFIG_ORDER = ["block_fp32", "d12", "d20_gqa", "d24", "d26_fp8"]


def config(name: str, **overrides) -> dict:
    """A copy of a preset with fields replaced (used to shrink B/T/L for tests)."""
    c = copy.deepcopy(CONFIGS[name])
    for k, v in overrides.items():
        c[k] = v
    L = c["n_layer"]
    if "window" not in overrides and len(c["window"]) != L:
        base = CONFIGS[name]["window"]
        c["window"] = [base[i % len(base)] for i in range(L)]
    if "has_ve" not in overrides and len(c["has_ve"]) != L:
        c["has_ve"] = _alternating_ve(L) if any(CONFIGS[name]["has_ve"]) else [0] * L
    if "backout_layer" not in overrides and CONFIGS[name]["backout_layer"] >= 0:
        c["backout_layer"] = L // 2
    return c


def qkv_width(c: dict) -> int:
    return (c["n_head"] + 2 * c["n_kv_head"]) * c["head_dim"]


# ---------------------------------------------------------------------------
# Random draws
# ---------------------------------------------------------------------------


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def round_to(x: torch.Tensor, dtype: str) -> torch.Tensor:
    """Round fp32 values to the storage dtype and return them as fp32."""
    if dtype == "f32":
        return x.float()
    return x.to(torch.bfloat16).float()


def normal(shape, std, g, dtype="bf16") -> torch.Tensor:
    return round_to(torch.randn(*shape, generator=g, dtype=torch.float32) * std, dtype)


def uniform(shape, lo, hi, g) -> torch.Tensor:
    return torch.rand(*shape, generator=g, dtype=torch.float32) * (hi - lo) + lo


def tokens(shape, vocab, g) -> torch.Tensor:
    return torch.randint(0, vocab, tuple(shape), generator=g, dtype=torch.int32)


def storage_dtype(c: dict) -> str:
    # FP8 configs keep bf16 storage; e4m3 appears only as GEMM operands
    return "f32" if c["dtype"] == "f32" else "bf16"


def make_weights(c: dict, seed: int = 1234, mode: str = "random", std: float = 0.02,
                 gate_std: float = 0.2) -> dict:
    """Seeded weights for a config.

    mode="init":   resid_lambda=1, x0_lambda=0, smear/backout lambdas 0.5
    mode="random": lambdas drawn away from the trivial values so that every
                   term contributes (resid U(0.5,1.5), x0 U(-0.5,0.5),
                   smear/backout U(0.2,0.8)); gate weights N(0, gate_std).
    Matrices are N(0, std) rounded to the storage dtype.  Returned tensors are
    fp32 CPU tensors (bf16-representable for bf16 storage); scalars are fp32.
    """
    g = _gen(seed)
    dt = storage_dtype(c)
    d, H, Hk, hd, F, V, L = (c["d"], c["n_head"], c["n_kv_head"], c["head_dim"],
                             c["mlp_hidden"], c["vocab"], c["n_layer"])
    w = {"layers": []}
    for i in range(L):
        lw = {
            "w_qkv": normal(((H + 2 * Hk) * hd, d), std, g, dt),
            "w_o": normal((d, H * hd), std, g, dt),
            "w_fc": normal((F, d), std, g, dt),
            "w_proj": normal((d, F), std, g, dt),
        }
        if mode == "random":
            lw["resid_lambda"] = float(uniform((1,), 0.5, 1.5, g)[0])
            lw["x0_lambda"] = float(uniform((1,), -0.5, 0.5, g)[0])
        else:
            lw["resid_lambda"], lw["x0_lambda"] = 1.0, 0.0
        if c["has_ve"][i]:
            lw["w_ve_gate"] = normal((Hk, c["ve_gate_ch"]), gate_std, g, dt)
            lw["ve_table"] = normal((V, Hk * hd), 1.0 if mode == "random" else std, g, dt)
        w["layers"].append(lw)
    if c.get("lm_head", True):
        w["wte"] = normal((V, d), 1.0 if mode == "random" else std, g, dt)
        w["w_lm"] = normal((V, d), std, g, dt)
    if c["smear_ch"] > 0:
        w["w_smear_gate"] = normal((c["smear_ch"],), gate_std, g, dt)
        w["smear_lambda"] = float(uniform((1,), 0.2, 0.8, g)[0]) if mode == "random" else 0.5
    if c["backout_layer"] >= 0:
        w["backout_lambda"] = float(uniform((1,), 0.2, 0.8, g)[0]) if mode == "random" else 0.5
    return w


def make_batch(c: dict, seed: int = 4321) -> dict:
    """Token ids and next-token targets, uniform in [0, vocab), int32 [B, T]."""
    g = _gen(seed)
    return {
        "idx": tokens((c["B"], c["T"]), c["vocab"], g),
        "targets": tokens((c["B"], c["T"]), c["vocab"], g),
    }


def make_block_inputs(c: dict, seed: int = 999, x_std: float = 1.0) -> dict:
    """Block-level inputs: x, x0 ~ N(0, x_std), upstream grad ~ N(0, 1), token ids."""
    g = _gen(seed)
    dt = storage_dtype(c)
    B, T, d = c["B"], c["T"], c["d"]
    return {
        "x": normal((B, T, d), x_std, g, dt),
        "x0": normal((B, T, d), x_std, g, dt),
        "dy": normal((B, T, d), 1.0, g, dt),
        "idx": tokens((B, T), c["vocab"], g),
    }
