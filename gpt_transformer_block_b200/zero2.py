"""Data-parallel optimizer step with ZeRO-2 sharding: the host orchestration.

Source: apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour 50€ ?",
§ "Comment nanochat fonctionne" › 2 "L'optimiseur Muon" › "Entraînement
distribué": the gradients are sharded ZeRO-2 style and the step runs in three
phases — (1) launch every asynchronous reduce_scatter, (2) wait for the
reductions, compute the updates, launch the all_gathers, (3) wait for the
gathers and copy the updated parameters back — so communication overlaps the
update computation.

Readings (the pages give the phases, not the sharding):
  - an AdamW parameter is flattened, padded to a multiple of 4 * world
    elements and split into `world` equal contiguous shards; rank r owns shard
    r and keeps the AdamW moments of that shard only;
  - a Muon matrix is not split (its Polar Express update needs the whole
    matrix): each is owned by one rank (largest first, to the least loaded
    rank); its reduce_scatter is a reduce to the owner and its all_gather a
    broadcast from the owner;
  - gradients are averaged over the ranks (sum, then divide by world).

The updates themselves are callables supplied by the caller: on the GPU the
library's gptb_adamw_step / gptb_polar_express kernels, in the CPU tests the
fp64 oracle.  Every rank issues the same collectives in the same order.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist


@dataclasses.dataclass
class ParamSpec:
    name: str
    shape: tuple
    kind: str  # "adamw" or "muon"

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= int(s)
        return n


class Zero2Plan:
    """Which rank owns what: shard extents of the AdamW parameters, owners of
    the Muon matrices.  Deterministic, so every rank builds the same plan."""

    def __init__(self, specs: list[ParamSpec], world: int):
        if world < 1:
            raise ValueError("world must be >= 1")
        self.specs = list(specs)
        self.world = world
        self.padded = {}
        self.owner = {}
        for s in self.specs:
            if s.kind == "adamw":
                q = 4 * world
                self.padded[s.name] = (s.numel + q - 1) // q * q
            elif s.kind != "muon":
                raise ValueError(f"unknown kind {s.kind!r} for {s.name}")
        load = [0] * world
        for s in sorted((s for s in self.specs if s.kind == "muon"), key=lambda s: (-s.numel, s.name)):
            r = min(range(world), key=lambda i: (load[i], i))
            self.owner[s.name] = r
            load[r] += s.numel
        self.muon_load = load

    def shard_len(self, name: str) -> int:
        return self.padded[name] // self.world

    def shard_range(self, name: str, rank: int) -> tuple:
        n = self.shard_len(name)
        return rank * n, (rank + 1) * n


def _has_native(group) -> bool:
    return dist.get_backend(group) == "nccl"


def _reduce_scatter(out, full, group, native):
    if native:
        return dist.reduce_scatter_tensor(out, full, op=dist.ReduceOp.SUM, group=group, async_op=True)
    # gloo has no reduce_scatter: all_reduce in place, the shard is sliced after the wait
    return dist.all_reduce(full, op=dist.ReduceOp.SUM, group=group, async_op=True)


def _all_gather(full, shard, group, native):
    if native:
        return dist.all_gather_into_tensor(full, shard, group=group, async_op=True)
    parts = list(full.chunk(dist.get_world_size(group)))
    return dist.all_gather(parts, shard.clone(), group=group, async_op=True), parts


def step(plan: Zero2Plan, params: dict, grads: dict, update_adamw, update_muon, group=None):
    """One data-parallel optimizer step in the three phases.

    params[name]: this rank's full parameter tensor (updated in place);
    grads[name]: this rank's local gradient (same shape; read, and used as a
    communication buffer); update_adamw(name, p_shard, g_shard) updates the
    1-D shard in place with the averaged gradient shard; update_muon(name, p,
    g) updates a whole matrix in place (called on its owner only)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if world != plan.world:
        raise ValueError("plan built for another world size")
    native = _has_native(group)
    # phase 1: every reduction goes out before any update
    pending = []
    for s in plan.specs:
        g = grads[s.name]
        if s.kind == "adamw":
            full = torch.zeros(plan.padded[s.name], dtype=g.dtype, device=g.device)
            full[: s.numel] = g.reshape(-1)
            shard = torch.empty(plan.shard_len(s.name), dtype=g.dtype, device=g.device)
            pending.append((s, _reduce_scatter(shard, full, group, native), full, shard))
        else:
            pending.append((s, dist.reduce(g, dst=plan.owner[s.name], op=dist.ReduceOp.SUM, group=group,
                                           async_op=True), g, None))
    # phase 2: wait for each reduction, update what this rank owns, launch the gathers
    gathers = []
    for s, work, buf, shard in pending:
        work.wait()
        p = params[s.name]
        if s.kind == "adamw":
            lo, hi = plan.shard_range(s.name, rank)
            if not native:
                shard.copy_(buf[lo:hi])
            shard.div_(world)
            pfull = torch.zeros(plan.padded[s.name], dtype=p.dtype, device=p.device)
            pfull[: s.numel] = p.reshape(-1)
            pshard = pfull[lo:hi].clone()
            update_adamw(s.name, pshard, shard)
            gathers.append((s, _all_gather(pfull, pshard, group, native), pfull))
        else:
            owner = plan.owner[s.name]
            if rank == owner:
                buf.div_(world)
                update_muon(s.name, p, buf)
            gathers.append((s, dist.broadcast(p, src=owner, group=group, async_op=True), None))
    # phase 3: wait for the gathers, copy the updated parameters back
    for s, work, pfull in gathers:
        if s.kind == "adamw":
            if native:
                work.wait()
            else:
                w, parts = work
                w.wait()
                pfull.copy_(torch.cat(parts))
            params[s.name].reshape(-1).copy_(pfull[: s.numel])
        else:
            work.wait()
