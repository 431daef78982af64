"""FSDP2-style sharded data parallelism whose collectives are TIDE's, one process per rank.

FSDP2 keeps every parameter as its own tensor and shards it along dim 0: rank r owns rows
[r*S, (r+1)*S) of each parameter, padded to W*S rows.  Stock FSDP2 all-gathers the shards
into a flat rank-major buffer and copies them out into the parameters, and packs each rank's
bf16 gradients into a flat fp32 buffer before the reduce-scatter (weekinpapers.com,
Abstract; kongchang.com, "The Root of FSDP2 Communication Overhead").  Here neither flat
buffer exists: TIDE-AG places every rank's shard straight into the parameters, and TIDE-RS
reduces each rank's shard straight from every rank's per-parameter gradients (same Abstract;
kongchang.com, "TIDE's Design Approach").  The ranks' buffers reach each other through CUDA
IPC (fsdp2_layout_aware_b200.exchange); the library's kernels read them directly.

A ``ShardedParams`` object owns, on this rank:
  * the full parameters' storage, padded to W*S_i rows (each parameter's ``data`` is a view
    of its first d0_i rows, so the module computes with the placed parameters in place);
  * a gradient arena: each parameter's ``grad`` is a view of it, so autograd accumulates the
    rank's gradients where the other ranks' reductions read them;
  * this rank's bf16 shard of every parameter (the shard arena, read by every rank's
    placement) and its fp32 master copy, which the optimizer updates.

A training step: ``unshard()`` before the forward, ``reduce_grads()`` after the backward (the
rank's fp32 gradient shard, x 1/W), ``sgd_step(lr)`` (or any update of ``master`` followed by
``publish()``), ``zero_grad()`` before the next backward.  Ranks meet only at host barriers
of the process group, placed so that no rank writes a buffer that another may still read:
before a placement (every rank's shard is current), after a reduction's start (every rank's
gradients are complete) and after its end (no rank clears its gradients while a peer reads
them).  This module moves no data itself: every byte moves in the library's kernels.
"""
from __future__ import annotations

from . import exchange as X
from . import tide as T


class ShardedParams:
    """One group of parameters trained data-parallel over the process group, dim-0 sharded.

    params: the module's parameters (bf16 CUDA tensors, the same values on every rank when
    the object is built).  They are re-pointed at storage this object owns.
    """

    def __init__(self, params, group=None, device=None):
        import torch
        import torch.distributed as dist

        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.params = list(params)
        if not self.params:
            raise ValueError("no parameters")
        for p in self.params:
            if p.dtype != torch.bfloat16 or not p.is_cuda or p.dim() == 0:
                raise ValueError("parameters must be bf16 CUDA tensors with at least one dim")
        dev = self.params[0].device if device is None else torch.device(device)
        self.device = dev
        W, r = self.world, self.rank
        shapes = [tuple(p.shape) for p in self.params]
        self.shapes = shapes
        self.plan = T.Plan(shapes, W, device=dev)                  # every rank's placement
        self.rank_plan = T.Plan(shapes, W, device=dev, rank=r)      # this rank's reduction
        Ns = self.plan.shard_numel
        self.shard_numel = Ns
        lay = X.arena_layout(shapes, W, W, Ns)                      # one rank per process
        self.layout = lay
        self.grad_arena = torch.zeros(lay.grad_elems, dtype=torch.bfloat16, device=dev)
        self.shard_arena = torch.zeros(lay.shard_elems, dtype=torch.bfloat16, device=dev)
        self.storage = []
        for i, p in enumerate(self.params):
            q = self.plan.query(i)
            st = torch.zeros(q["padded_numel"], dtype=torch.bfloat16, device=dev)
            n = p.numel()
            st[:n].copy_(p.detach().reshape(-1))
            self.storage.append(st)
            with torch.no_grad():
                p.data = st[:n].view(p.shape)
            o = lay.grad_off[i]
            p.grad = self.grad_arena[o: o + n].view(p.shape)
        # this rank's shard of every parameter: rows [r*S_i, (r+1)*S_i), pad rows zero
        self.shard = self.shard_arena[:Ns]
        for i in range(len(self.params)):
            q = self.plan.query(i)
            c, off = q["chunk_numel"], q["shard_offset"]
            self.shard[off: off + c].copy_(self.storage[i][r * c: (r + 1) * c])
        self.master = self.shard.float()                            # fp32 master shard
        self.grad_shard = torch.zeros(Ns, dtype=torch.float32, device=dev)
        torch.cuda.synchronize(dev)
        dist.barrier(group)                                         # every rank's arenas exist
        local = {"grads": self.grad_arena.data_ptr(), "shards": self.shard_arena.data_ptr()}
        exports = X.all_exports(X.export({"grads": self.grad_arena, "shards": self.shard_arena}), group)
        self.peers = X.PeerMaps(exports, r, dev.index, local)
        gp, gn = X.grad_table(lay, W, W, self.peers.bases("grads", W))
        self.grad_table = T.PointerTable(gp, gn, keep=[self.grad_arena])
        self.shard_table = T.PointerTable(X.shard_table(lay, W, W, self.peers.bases("shards", W)),
                                          [Ns] * W, keep=[self.shard_arena])
        self.storage_table = T.TensorTable(self.storage)

    def _meet(self):
        import torch
        import torch.distributed as dist
        torch.cuda.synchronize(self.device)
        dist.barrier(self.group)

    def unshard(self, engine: int = T.TIDE_ENGINE_SM) -> None:
        """Place every rank's shard into this rank's full parameters (TIDE-AG)."""
        self._meet()                                                # every rank's shard is current
        self.plan.ag_gather_place(self.shard_table, self.storage_table, engine=engine)

    def reduce_grads(self, order: int = T.TIDE_ORDER_RANK) -> None:
        """This rank's fp32 gradient shard, x fl32(1/W), from every rank's gradients (TIDE-RS)."""
        self._meet()                                                # every rank's gradients are done
        self.rank_plan.rs_reduce(self.grad_table, self.grad_shard,
                                 scale_mode=T.TIDE_SCALE_INV_WORLD, order=order)
        self._meet()                                                # no rank clears them while read

    def zero_grad(self) -> None:
        self.grad_arena.zero_()

    def publish(self) -> None:
        """Round the fp32 master shard into the bf16 shard the other ranks place from."""
        self.shard.copy_(self.master)

    def sgd_step(self, lr: float) -> None:
        """master -= lr * grad_shard (fp32), then publish.  Pad positions stay zero."""
        self.master.add_(self.grad_shard, alpha=-lr)
        self.publish()

    def close(self) -> None:
        """Unmap the peers' arenas once no rank can still read them."""
        if getattr(self, "peers", None) is not None:
            self._meet()
            self.peers.close()
            self._meet()
            self.peers = None
