"""Device-memory holders around the C ABI (PyTorch allocates; the library computes).

GPTStack   weights, fp32 gradient buffers and the step workspace of a whole
           stack; ``step(idx, targets)`` enqueues one gpt_stack_step.
BlockRunner one block's saved-activation and scratch workspaces for
           gpt_block_forward / gpt_block_backward.
"""
from __future__ import annotations

import torch

from . import (BF16, F32, WS_BLOCK_SAVED, WS_BLOCK_SCRATCH, WS_LM_HEAD, WS_STACK, block_grads,
               block_weights, gpt_block_backward, gpt_block_forward, gpt_stack_step, gptb_workspace_bytes,
               lm_head_xent, make_config, model_grads, model_weights)


def storage_torch_dtype(c: dict) -> torch.dtype:
    return torch.float32 if c["dtype"] == "f32" else torch.bfloat16


def to_device_weights(c: dict, w: dict, device="cuda") -> dict:
    """Copy synthetic (CPU fp32) weights to the device in the storage dtype."""
    dt = storage_torch_dtype(c)

    def mat(t):
        return t.to(device=device, dtype=dt).contiguous()

    out = {"layers": []}
    for lw in w["layers"]:
        d = {k: mat(lw[k]) for k in ("w_qkv", "w_o", "w_fc", "w_proj")}
        d["lambdas"] = torch.tensor([lw["resid_lambda"], lw["x0_lambda"]], dtype=torch.float32, device=device)
        if "w_ve_gate" in lw:
            d["w_ve_gate"] = mat(lw["w_ve_gate"])
            d["ve_table"] = mat(lw["ve_table"])
        out["layers"].append(d)
    for k in ("wte", "w_lm", "w_smear_gate"):
        if k in w:
            out[k] = mat(w[k])
    for k in ("smear_lambda", "backout_lambda"):
        if k in w:
            out[k] = torch.tensor([w[k]], dtype=torch.float32, device=device)
    return out


def zero_grads_like(c: dict, dw: dict) -> dict:
    """fp32 gradient buffers matching the device weights."""
    g = {"layers": []}
    for lw in dw["layers"]:
        g["layers"].append({k: torch.zeros(v.shape, dtype=torch.float32, device=v.device) for k, v in lw.items()})
    for k in ("wte", "w_lm", "w_smear_gate", "smear_lambda", "backout_lambda"):
        if k in dw:
            g[k] = torch.zeros(dw[k].shape, dtype=torch.float32, device=dw[k].device)
    return g


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


class GPTStack:
    """One stack's weights, gradients and step workspace on the current device."""

    def __init__(self, c: dict, weights: dict, device="cuda"):
        self.c = c
        self.cfg = make_config(c)
        self.device = torch.device(device)
        self.w = to_device_weights(c, weights, device)
        self.g = zero_grads_like(c, self.w)
        self.ws = _ws(gptb_workspace_bytes(self.cfg, WS_STACK), self.device)
        self.loss = torch.zeros(1, dtype=torch.float32, device=self.device)
        self._mw = model_weights(self.w)
        self._mg = model_grads(self.g)

    def zero_grad(self):
        for lg in self.g["layers"]:
            for v in lg.values():
                v.zero_()
        for k, v in self.g.items():
            if k != "layers":
                v.zero_()

    def step(self, idx: torch.Tensor, targets: torch.Tensor, stream=None) -> torch.Tensor:
        """Forward + backward of the whole stack; grads accumulate; returns the loss tensor."""
        gpt_stack_step(self.cfg, self._mw, idx, targets, self.loss, self._mg, self.ws, stream)
        return self.loss


class BlockRunner:
    """Workspaces for one block's forward/backward through the C ABI."""

    def __init__(self, c: dict, device="cuda"):
        self.c = c
        self.cfg = make_config(c)
        self.device = torch.device(device)
        self.saved = _ws(gptb_workspace_bytes(self.cfg, WS_BLOCK_SAVED), self.device)
        self.scratch = _ws(gptb_workspace_bytes(self.cfg, WS_BLOCK_SCRATCH), self.device)

    def forward(self, layer, lw: dict, x, x0, idx, x_out, stream=None):
        gpt_block_forward(self.cfg, layer, block_weights(lw), x, x0, idx, x_out, self.saved, self.scratch, stream)

    def backward(self, layer, lw: dict, x, x0, idx, dx_out, dx, dx0_accum, lg: dict, dx_extra=None,
                 stream=None):
        gpt_block_backward(self.cfg, layer, block_weights(lw), x, x0, idx, self.saved, dx_out, dx_extra, dx,
                           dx0_accum, block_grads(lg), self.scratch, stream)


def lm_head(c: dict, h, w_lm, targets, dh, dw_lm, stream=None):
    """lm_head_xent through the C ABI with a fresh workspace; returns the loss tensor."""
    cfg = make_config(c)
    ws = _ws(gptb_workspace_bytes(cfg, WS_LM_HEAD), h.device)
    loss = torch.zeros(1, dtype=torch.float32, device=h.device)
    lm_head_xent(cfg, h, w_lm, targets, loss, dh, dw_lm, ws, stream)
    return loss


__all__ = ["GPTStack", "BlockRunner", "to_device_weights", "zero_grads_like", "lm_head", "BF16", "F32"]
