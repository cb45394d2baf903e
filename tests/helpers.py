"""Shared helpers for the parity tests (no method arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

import synth

TOL = {"bf16": 2e-2, "fp8": 6e-2, "f32": 1e-5}


def relerr(gpu, ref) -> float:
    """Normwise max relative error: max|gpu - ref| / max|ref|."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    denom = np.max(np.abs(r)) if r.size else 0.0
    if denom == 0.0:
        return float(np.max(np.abs(g))) if g.size else 0.0
    return float(np.max(np.abs(g - r)) / denom)


def scalar_err(gpu: float, ref: float, scale: float) -> float:
    """Error of a scalar sum judged against the sum of its terms' magnitudes
    (forward-error bound of a rounded dot product): |gpu - ref| / sum|terms|."""
    return abs(float(gpu) - float(ref)) / max(float(scale), 1e-300)


def fp8_mode(c: dict):
    """The oracle's fp8 argument for a config: False, True (e4m3 operands) or
    "e5m2" (e5m2 gradient operands)."""
    if c["dtype"] != "fp8":
        return False
    return "e5m2" if c.get("fp8_grad") == "e5m2" else True


def np64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def oracle_layer(w: dict, i: int) -> dict:
    """Synthetic layer weights as fp64 numpy arrays / floats for the oracle."""
    out = {}
    for k, v in w["layers"][i].items():
        out[k] = v if isinstance(v, float) else np64(v)
    return out


def oracle_weights(w: dict) -> dict:
    out = {"layers": [oracle_layer(w, i) for i in range(len(w["layers"]))]}
    for k, v in w.items():
        if k != "layers":
            out[k] = v if isinstance(v, float) else np64(v)
    return out


def small_bf16(**kw) -> dict:
    """A small bf16 stack that spans several GEMM tiles with ragged tails."""
    base = dict(B=2, T=200, d=256, n_head=2, n_kv_head=1, n_layer=3, vocab=512, mlp_hidden=1024,
                window=[-1, 48, -1], has_ve=[0, 1, 0], backout_layer=1)
    base.update(kw)
    return synth.config("d24", **base)


# FP8 parity.  An FP8 product quantises bf16 tensors; the GPU and the
# FP8-emulating oracle reach those tensors by different roundings (fp32 vs
# fp64 upstream), so an e4m3 code near a rounding boundary can differ (one
# code = 12.5 %).  Quantities made mostly of FP8 products (weight gradients,
# gradients that crossed several FP8 layers) therefore differ from the
# oracle's by the FP8 noise itself.  Such a quantity passes when it is within
# the tolerance of the FP8 oracle, or when it is as close to the exact
# (non-FP8) result as the FP8 oracle's own value is (within FP8_ENVELOPE
# times that distance): a valid FP8 evaluation of the same inputs.  A wrong
# scale, operand or index fails both.
FP8_ENVELOPE = 1.5


def judge(errs: dict, tol: float, gpu_exact: dict | None = None, ref_exact: dict | None = None) -> dict:
    """The entries of errs (GPU vs the reference of its configuration) above
    tol that, for FP8, are also outside the envelope; {} when all pass."""
    bad = {}
    for k, e in errs.items():
        if e <= tol:
            continue
        if gpu_exact is not None and gpu_exact[k] <= FP8_ENVELOPE * ref_exact[k]:
            continue
        bad[k] = (e, gpu_exact.get(k) if gpu_exact else None, ref_exact.get(k) if ref_exact else None)
    return bad
