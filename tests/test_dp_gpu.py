"""The ZeRO-2 data-parallel step on the GPU (GpuZero2Trainer) at world size 1
on NCCL, so that the native reduce_scatter / all_gather / reduce / broadcast
branch, the bf16 gradient buckets launched from the gradients-ready hook of
gpt_stack_step_hooked, and the library's AdamW and Muon kernels on the
owned shards all run.  Checked against the same optimizer kernels applied to
whole tensors without the data-parallel machinery (with world size 1 the
averaged gradient is the bf16 rounding of the rank's own gradient).  The
two-rank orchestration is tested on gloo on the CPU (test_zero2.py)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

import synth
from helpers import TOL, relerr, small_bf16
from oracle import optim as oo

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_zero2_trainer_world1_matches_direct_updates(cuda_lib):
    """After one trainer step every parameter equals the optimizer kernels
    applied directly to its pre-step value and the bf16 rounding of the
    gradient the step produced (the trainer's own gradient: the reductions'
    fp32 atomics are unordered, and the orthogonalisation amplifies
    near-null directions of the gradient about 1000-fold, so two separate
    gradient evaluations are not comparable this way)."""
    gb = cuda_lib
    from gpt_transformer_block_b200.model import GPTStack
    from gpt_transformer_block_b200.zero2 import GpuZero2Trainer, stack_param_specs
    c = small_bf16(n_layer=2, window=[-1, 32], has_ve=[0, 1], backout_layer=1)
    w = synth.make_weights(c, seed=61)
    b = synth.make_batch(c, seed=62)
    idx, tg = b["idx"].cuda(), b["targets"].cuda()
    hp = dict(lr_adamw=3e-3, betas=(0.8, 0.95), eps=1e-10, lr_muon=0.02, momentum=0.95, beta2_muon=0.95,
              weight_decay=0.01)
    coeffs = oo.POLAR_EXPRESS_COEFFS
    ref = GPTStack(c, w)
    ref.step(idx, tg)
    torch.cuda.synchronize()
    loss_ref = ref.loss.item()

    os.environ["NCCL_NVLS_ENABLE"] = "0"
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        tr = GpuZero2Trainer(c, w, **hp, coeffs=coeffs)
        specs = stack_param_specs(c)
        before = {s.name: tr.param(s.name).clone() for s in specs}
        loss, order = tr.step(idx, tg)
        torch.cuda.synchronize()
        assert gb.gptb_device_error() == 0
        assert order == [1, 0, -1]
        assert abs(loss.item() - loss_ref) <= 1e-5 * abs(loss_ref)
        for s in specs:
            p0 = before[s.name]
            g = tr.grad(s.name).bfloat16().float().contiguous()
            master = p0.float().contiguous().clone()
            if s.kind == "adamw":
                n = master.numel()
                pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
                gb.gptb_adamw_step(master, g, torch.zeros_like(master), torch.zeros_like(master), pb, n,
                                   hp["lr_adamw"], hp["betas"][0], hp["betas"][1], hp["eps"], hp["weight_decay"], 1)
                want = (pb if p0.dtype == torch.bfloat16 else master).reshape(p0.shape)
                torch.cuda.synchronize()
                assert torch.equal(tr.param(s.name), want), s.name
            else:
                m, n = s.shape
                pb = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
                ws = torch.empty(gb.gptb_muon_workspace_bytes(m, n, len(coeffs)), dtype=torch.uint8, device="cuda")
                gb.gptb_muon_step(master, pb, g, torch.zeros_like(master), torch.zeros(m, device="cuda"), m, n,
                                  coeffs, hp["lr_muon"], hp["momentum"], hp["beta2_muon"], hp["weight_decay"], ws)
                torch.cuda.synchronize()
                st = tr.state[s.name]
                # the reduced bf16 gradient reached the Muon step: with a zero
                # buffer the momentum update leaves exactly that gradient
                assert torch.equal(st["buf"], g), s.name
                # NorMuon's two sums are float atomics, so the fp32 masters may
                # differ in the last bits; the update they received agrees to
                # far below the bf16 tolerance
                err = relerr((st["master"] - p0.float()).double().cpu().numpy(),
                             (master - p0.float()).double().cpu().numpy())
                assert err <= 1e-4, (s.name, err)
                # and the bf16 working weight is the rounding of the trainer's own
                # master (a last-bit master difference may move that rounding by
                # one step against the direct call's, so it is not compared)
                assert torch.equal(tr.param(s.name), st["master"].bfloat16()), s.name
    finally:
        dist.destroy_process_group()


def _get(tree, name):
    if name.startswith("L"):
        i, k = name.split(".", 1)
        return tree["layers"][int(i[1:])][k]
    return tree[name]
