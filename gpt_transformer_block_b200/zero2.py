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

`step` takes the updates as callables (in the CPU tests the fp64 oracle);
GpuZero2Trainer below runs the same phases on the GPU with the library's
gptb_adamw_step / gptb_muon_step kernels, bf16 gradient buckets launched per
layer from inside the backward, and NCCL.  Every rank issues the same
collectives in the same order.
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


# ---------------------------------------------------------------------------
# The same three phases on the GPU library, with per-layer buckets launched
# from inside the backward.
# ---------------------------------------------------------------------------

def stack_param_specs(c: dict) -> list[ParamSpec]:
    """Parameters of a stack with their optimizer ([JA-opt] on the source pages:
    AdamW for the embeddings, the lm_head and the scalars, Muon for the 2-D
    matrices).  Reading: the Muon matrices are the four block projections;
    the value-embedding tables, the small gate weights and every lambda take
    AdamW.  Names are "L<i>.<weight>" for block weights."""
    specs = []
    d, H, Hk, hd, F, V = c["d"], c["n_head"], c["n_kv_head"], c["head_dim"], c["mlp_hidden"], c["vocab"]
    for i in range(c["n_layer"]):
        specs += [ParamSpec(f"L{i}.w_qkv", ((H + 2 * Hk) * hd, d), "muon"), ParamSpec(f"L{i}.w_o", (d, H * hd), "muon"),
                  ParamSpec(f"L{i}.w_fc", (F, d), "muon"), ParamSpec(f"L{i}.w_proj", (d, F), "muon"),
                  ParamSpec(f"L{i}.lambdas", (2,), "adamw")]
        if c["has_ve"][i]:
            specs += [ParamSpec(f"L{i}.w_ve_gate", (Hk, c["ve_gate_ch"]), "adamw"),
                      ParamSpec(f"L{i}.ve_table", (V, Hk * hd), "adamw")]
    specs += [ParamSpec("wte", (V, d), "adamw"), ParamSpec("w_lm", (V, d), "adamw")]
    if c["smear_ch"] > 0:
        specs += [ParamSpec("w_smear_gate", (c["smear_ch"],), "adamw"), ParamSpec("smear_lambda", (1,), "adamw")]
    if c["backout_layer"] >= 0:
        specs.append(ParamSpec("backout_lambda", (1,), "adamw"))
    return specs


class GpuZero2Trainer:
    """One data-parallel training step per call on this rank's batch:

    - the stack step (gpt_stack_step_hooked); as each layer's gradients are
      enqueued, its bucket is cast to bf16 (1/world folded in) on a
      communication stream after an event on the compute stream, and its
      reductions start there (reduce_scatter for AdamW tensors, reduce to the
      owner for Muon matrices), overlapping the rest of the backward
      (phase 1);
    - each reduction is waited for, the owned AdamW shards updated by
      gptb_adamw_step and their all_gather launched; the owned Muon matrices
      are updated by one gptb_muon_step_batched call per shape (fp32 masters
      that write the bf16 working weights), then every rank launches the
      Muon broadcasts in the same order (phase 2);
    - the gathers are waited for and the working weights filled (phase 3).

    Masters and optimizer state exist only for what this rank owns (ZeRO-2).
    NCCL only (bf16 collectives, reduce_scatter); the orchestration itself is
    `step` above, tested on gloo on the CPU."""

    def __init__(self, c: dict, weights: dict, group=None, lr_adamw=3e-4, betas=(0.8, 0.95), eps=1e-10,
                 lr_muon=0.02, momentum=0.95, beta2_muon=0.95, weight_decay=0.0, coeffs=None):
        from . import model as gm
        import gpt_transformer_block_b200 as gb
        if coeffs is None:
            raise ValueError("pass the Polar Express coefficient tuples")
        self.gb = gb
        self.c = c
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.stack = gm.GPTStack(c, weights)
        self.specs = stack_param_specs(c)
        self.plan = Zero2Plan(self.specs, self.world)
        self.hp = dict(lr_adamw=lr_adamw, betas=betas, eps=eps, lr_muon=lr_muon, momentum=momentum,
                       beta2_muon=beta2_muon, weight_decay=weight_decay)
        self.coeffs = [tuple(float(x) for x in t) for t in coeffs]
        self.t = 0
        self.comm = torch.cuda.Stream()
        dev = self.stack.device
        self.by_layer = {}
        for s in self.specs:
            layer = int(s.name.split(".")[0][1:]) if s.name.startswith("L") else -1
            self.by_layer.setdefault(layer, []).append(s)
        # bf16 communication buffers and this rank's optimizer state
        self.wire, self.state = {}, {}
        for s in self.specs:
            p = self.param(s.name)
            if s.kind == "adamw":
                n = self.plan.shard_len(s.name)
                lo, hi = self.plan.shard_range(s.name, self.rank)
                full = torch.zeros(self.plan.padded[s.name], dtype=torch.float32, device=dev)
                full[: s.numel] = p.reshape(-1).float()
                self.wire[s.name] = (torch.zeros(self.plan.padded[s.name], dtype=torch.bfloat16, device=dev),
                                     torch.zeros(n, dtype=torch.bfloat16, device=dev))
                # the gather carries the parameter's own dtype: bf16 working
                # copies, or the fp32 masters of the fp32 scalars
                self.state[s.name] = dict(master=full[lo:hi].clone(), m=torch.zeros(n, device=dev),
                                          v=torch.zeros(n, device=dev), g=torch.zeros(n, device=dev),
                                          pb=torch.zeros(n, dtype=torch.bfloat16, device=dev),
                                          gathered=torch.zeros(self.plan.padded[s.name], dtype=p.dtype, device=dev))
            else:
                self.wire[s.name] = (torch.zeros(s.shape, dtype=torch.bfloat16, device=dev), None)
                if self.plan.owner[s.name] == self.rank:
                    m, n = s.shape
                    self.state[s.name] = dict(master=p.float().clone(), buf=torch.zeros(s.shape, device=dev),
                                              v=torch.zeros(m, device=dev), g=torch.zeros(s.shape, device=dev))
        # the owned Muon matrices by shape: each group takes one batched Muon call
        # (every Polar Express product one GEMM launch over the group)
        self.muon_groups = {}
        for s in self.specs:
            if s.kind != "adamw" and self.plan.owner[s.name] == self.rank:
                self.muon_groups.setdefault(tuple(s.shape), []).append(s)
        self.muon_ws = {shape: torch.empty(gb.gptb_muon_batched_workspace_bytes(len(grp), shape[0], shape[1],
                                                                                 len(self.coeffs)),
                                           dtype=torch.uint8, device=dev)
                        for shape, grp in self.muon_groups.items()}

    def _lookup(self, tree: dict, name: str):
        if name.startswith("L"):
            i, k = name.split(".", 1)
            lw = tree["layers"][int(i[1:])]
            return lw[k]
        return tree[name]

    def param(self, name):  # the bf16 working weight (fp32 for the scalars)
        return self._lookup(self.stack.w, name)

    def grad(self, name):   # the library's fp32 gradient
        return self._lookup(self.stack.g, name)

    def step(self, idx, targets):
        gb = self.gb
        self.t += 1
        self.stack.zero_grad()
        compute = torch.cuda.current_stream()
        pending = []
        order = []

        def ready(layer):
            order.append(layer)
            ev = torch.cuda.Event()
            ev.record(compute)
            with torch.cuda.stream(self.comm):
                self.comm.wait_event(ev)
                for s in self.by_layer.get(layer, []):
                    full, shard = self.wire[s.name]
                    gb.gptb_cast_f32_bf16(self.grad(s.name), full, s.numel, 1.0 / self.world, self.comm)
                    if s.kind == "adamw":
                        w = dist.reduce_scatter_tensor(shard, full, op=dist.ReduceOp.SUM, group=self.group,
                                                       async_op=True)
                    else:
                        w = dist.reduce(full, dst=self.plan.owner[s.name], op=dist.ReduceOp.SUM, group=self.group,
                                        async_op=True)
                    pending.append((s, w))

        gb.gpt_stack_step_hooked(self.stack.cfg, self.stack._mw, idx, targets, self.stack.loss, self.stack._mg,
                                 self.stack.ws, ready, compute)
        hp = self.hp
        gathers = []
        for s, w in pending:                     # phase 2: AdamW shards, and the owned Muon gradients in fp32
            w.wait()
            full, shard = self.wire[s.name]
            st = self.state.get(s.name)
            if s.kind == "adamw":
                gb.gptb_cast_bf16_f32(shard, st["g"], shard.numel(), 1.0, compute)
                gb.gptb_adamw_step(st["master"], st["g"], st["m"], st["v"], st["pb"], shard.numel(),
                                   hp["lr_adamw"], hp["betas"][0], hp["betas"][1], hp["eps"], hp["weight_decay"],
                                   self.t, compute)
                src = st["pb"] if st["gathered"].dtype == torch.bfloat16 else st["master"]
                gathers.append((s, dist.all_gather_into_tensor(st["gathered"], src, group=self.group,
                                                               async_op=True)))
            elif self.plan.owner[s.name] == self.rank:
                gb.gptb_cast_bf16_f32(full, st["g"], s.numel, 1.0, compute)
        for (m, n), grp in self.muon_groups.items():
            sts = [self.state[x.name] for x in grp]
            gb.gptb_muon_step_batched([x["master"] for x in sts], [self.param(x.name) for x in grp],
                                      [x["g"] for x in sts], [x["buf"] for x in sts], [x["v"] for x in sts], m, n,
                                      self.coeffs, hp["lr_muon"], hp["momentum"], hp["beta2_muon"],
                                      hp["weight_decay"], self.muon_ws[(m, n)], compute)
        for s, _ in pending:                     # every rank broadcasts the Muon matrices in the same order
            if s.kind != "adamw":
                gathers.append((s, dist.broadcast(self.param(s.name), src=self.plan.owner[s.name],
                                                  group=self.group, async_op=True)))
        for s, w in gathers:                     # phase 3
            w.wait()
            if s.kind == "adamw":
                self.param(s.name).reshape(-1).copy_(self.state[s.name]["gathered"][: s.numel])
        return self.stack.loss, order
