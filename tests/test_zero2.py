"""ZeRO-2 optimizer-step orchestration (gpt_transformer_block_b200/zero2.py)
on two gloo ranks on the CPU: after one step every rank holds exactly the
parameters a single process computes from the averaged gradients (AdamW by
the fp64 oracle on whole tensors, Polar Express by the oracle on whole
matrices), with padding-ragged AdamW tensors and Muon matrices of several
shapes; plus the plan's sharding and ownership rules."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gpt_transformer_block_b200.zero2 import ParamSpec, Zero2Plan

PAGE_TUPLES = [(8.156, -22.483, 15.879), (4.043, -2.809, 0.500)]
SPECS = [ParamSpec("wte", (37, 5), "adamw"), ParamSpec("w_qkv", (16, 8), "muon"),
         ParamSpec("lam", (1,), "adamw"), ParamSpec("w_proj", (8, 24), "muon"), ParamSpec("w_o", (8, 8), "muon")]
HP = dict(lr=1e-2, beta1=0.8, beta2=0.95, eps=1e-10, weight_decay=0.1)
MUON_LR = 0.02


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(world):
    rng = np.random.default_rng(7)
    params = {s.name: rng.standard_normal(s.shape) for s in SPECS}
    grads = [{s.name: rng.standard_normal(s.shape) for s in SPECS} for _ in range(world)]
    return params, grads


def _reference(world):
    from oracle import optim as oo
    params, grads = _inputs(world)
    out = {}
    for s in SPECS:
        g = sum(gr[s.name] for gr in grads) / world
        if s.kind == "adamw":
            out[s.name], _, _ = oo.adamw_step(params[s.name], g, np.zeros(s.shape), np.zeros(s.shape), 1, HP["lr"],
                                              HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"])
        else:
            out[s.name] = params[s.name] - MUON_LR * oo.polar_express(g, PAGE_TUPLES)
    return out


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from oracle import optim as oo
    from gpt_transformer_block_b200 import zero2
    plan = zero2.Zero2Plan(SPECS, world)
    params, grads = _inputs(world)
    P = {k: torch.tensor(v) for k, v in params.items()}
    G = {k: torch.tensor(v) for k, v in grads[rank].items()}
    state = {s.name: (np.zeros(plan.shard_len(s.name)), np.zeros(plan.shard_len(s.name)))
             for s in SPECS if s.kind == "adamw"}
    calls = []

    def upd_adamw(name, p, g):
        m, v = state[name]
        pn, m, v = oo.adamw_step(p.numpy(), g.numpy(), m, v, 1, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"],
                                 HP["weight_decay"])
        state[name] = (m, v)
        p.copy_(torch.tensor(pn))

    def upd_muon(name, p, g):
        calls.append(name)
        p.sub_(MUON_LR * torch.tensor(oo.polar_express(g.numpy(), PAGE_TUPLES)))

    zero2.step(plan, P, G, upd_adamw, upd_muon)
    out[rank] = ({k: v.numpy() for k, v in P.items()}, calls)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_step_equals_single_process():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    ref = _reference(world)
    plan = Zero2Plan(SPECS, world)
    for r in range(world):
        got, calls = out[r]
        for s in SPECS:
            # the padded tail of an AdamW shard sees zero gradient and zero parameter: it stays zero and is dropped
            assert np.allclose(got[s.name], ref[s.name], rtol=0, atol=1e-12), (r, s.name)
        # each Muon matrix is updated by its owner only
        assert sorted(calls) == sorted(n for n, o in plan.owner.items() if o == r)


def test_plan_shards_and_owners():
    plan = Zero2Plan(SPECS, 3)
    assert plan.padded["wte"] == 192 and plan.shard_len("wte") == 64   # 185 -> multiple of 12
    assert plan.padded["lam"] == 12 and plan.shard_range("lam", 2) == (8, 12)
    # largest matrix first, each to the least-loaded rank
    assert plan.owner == {"w_proj": 0, "w_qkv": 1, "w_o": 2}  # 192, 128, 64 elements
    with pytest.raises(ValueError):
        Zero2Plan([ParamSpec("x", (2,), "sgd")], 2)
