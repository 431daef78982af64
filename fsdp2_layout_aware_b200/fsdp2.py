"""TIDE's collectives inside FSDP2's own ``fully_shard``, one process per rank.

Around its collectives stock FSDP2 runs two layout conversions (weekinpapers.com, Abstract;
kongchang.com, "The Root of FSDP2 Communication Overhead"):
  * all-gather: each rank copies its bf16 shard into row r of a flat [W][Ns] buffer, the
    buffer is all-gathered, and a copy-out (``fsdp::split_with_sizes_copy``) splits it into
    the unsharded parameters;
  * reduce-scatter: each rank packs its bf16 gradients into a flat fp32 [W][Ns] buffer
    (``fsdp::chunk_cat``), which is reduce-scattered.
TIDE folds the copy-out into the all-gather's addressing and replaces the fp32 pack with
gradients read where they are, staged bf16 into the vacated all-gather slot under Slot-Reuse
(same Abstract; kongchang.com, "TIDE's Design Approach").  ``fully_shard_tide`` applies
``fully_shard`` and then, for the module's parameter group:
  * ``TideAllGather`` (``set_custom_all_gather``): the [W][Ns] buffer FSDP2 asks for is a
    persistent bf16 arena of this rank, mapped into every other rank through CUDA IPC.
    FSDP2's own copy-in writes this rank's row; the collective itself only waits until every
    rank's row is in place.  FSDP2's copy-out on that arena becomes ``tide_ag_gather_place``:
    row k read from rank k's arena and placed straight into the unsharded parameters, pad
    rows zeroed.  No rank ever holds the gathered [W][Ns] buffer.
  * ``TideReduceScatter`` (``set_custom_reduce_scatter``): the fp32 [W][Ns] input FSDP2 asks
    for is one element expanded to that shape, never written.  FSDP2's pack on it becomes
    ``tide_rs_stage_one``: this rank's bf16 gradients staged into its arena (the all-gather
    slot, free once every rank has placed from it).  The collective is
    ``tide_rs_reduce_slots`` with this rank's one-rank plan: its fp32 shard reduced in rank
    order from rows r of every rank's arena, x fl32(1/W) for FSDP2's average.
The copy-out and the pack are replaced through their dispatcher entries: on a buffer of a
TIDE group the library call runs; on any other buffer FSDP2's own implementation does.

Ranks meet only at host barriers of the process group (wait for this rank's stream, then
barrier), placed so
that no rank writes its arena while another may still read it: before a placement (every
row is in), after it (before anyone stages gradients over its row), before a reduction
(every rank staged) and after it (before the next copy-in).  The parameter group must have
bf16 compute parameters and fp32 reduction (the mixed-precision policy set here); every
collective is synchronous.  Parameters without a gradient (frozen ones) are left out of
FSDP2's reduce-scatter; the layout of the ones that have one follows from their shapes in
group order, and the group builds plans for that subset on first use.  Gradient
accumulation works both ways: with gradient sync on, every micro-batch is reduce-scattered and
FSDP2 sums the fp32 shards; with it off, FSDP2 keeps the unsharded gradients in fp32 and packs
those at the synced backward, which become ``tide_rs_stage_one_f32`` into a fp32 slot of the
rank (made on first use, W*Ns*4 bytes, the size of stock FSDP2's packed buffer) and
``tide_rs_reduce_slots_f32`` (rank order).
"""
from __future__ import annotations

import math
import threading
import warnings

from . import exchange as X
from . import tide as T

_AG = {}          # data_ptr of a group's arena -> TideGroup
_RS = {}          # data_ptr of a group's expanded reduce-scatter input -> TideGroup
_LOCK = threading.Lock()
_INSTALLED = set()   # dispatch keys whose copy-out and pack are routed here
_LIBS = []


def _check_grads(grads, n_params) -> bool:
    """Refuse what TIDE's staging cannot take: more gradients than parameters, or gradients
    that are not all contiguous bf16 or all contiguous fp32.  FSDP2 hands over fp32 gradients
    when they were accumulated with gradient sync off (it keeps those in the fp32 reduce
    dtype).  Returns True for fp32 gradients."""
    import torch
    if not 0 < len(grads) <= n_params:
        raise ValueError("gradients do not match the group's parameters")
    dtype = grads[0].dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("TIDE staging takes bf16 or fp32 gradients")
    for g in grads:
        if g.dtype != dtype or not g.is_contiguous() or g.dim() == 0:
            raise ValueError("TIDE staging takes the parameters' contiguous gradients, all of "
                             "one dtype")
    return dtype == torch.float32


class TideGroup:
    """The TIDE state of one FSDP2 parameter group on this rank.

    shapes: the group's unsharded parameter shapes in FSDP2's order.  Every rank builds its
    groups in the same order (the handle exchange is a collective).
    """

    def __init__(self, shapes, group=None, device=None, engine: int = T.TIDE_ENGINE_SM,
                 order: int = T.TIDE_ORDER_RANK):
        import torch
        import torch.distributed as dist

        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if self.world < 2:
            raise ValueError("TIDE's collectives need at least 2 ranks")
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.engine, self.order = engine, order
        W, r = self.world, self.rank
        self.shapes = [tuple(int(d) for d in s) for s in shapes]
        self.plan = T.Plan(self.shapes, W, device=self.device)             # placement, staging
        self.rank_plan = T.Plan(self.shapes, W, device=self.device, rank=r)  # this rank's shard
        Ns = self.plan.shard_numel
        self.shard_numel = Ns
        self.chunks = [self.plan.query(i)["chunk_numel"] for i in range(len(self.shapes))]
        self.arena = torch.zeros(W * Ns, dtype=torch.bfloat16, device=self.device)
        self.rs_input = torch.zeros(1, dtype=torch.float32, device=self.device)
        torch.cuda.synchronize(self.device)
        exports = X.all_exports(X.export({"arena": self.arena}), group)
        self.peers = X.PeerMaps(exports, r, self.device.index, {"arena": self.arena.data_ptr()})
        bases = self.peers.bases("arena", W)
        # row k of rank k's arena is rank k's shard; the slots are the whole arenas
        self.shard_table = T.PointerTable([b + 2 * k * Ns for k, b in enumerate(bases)], [Ns] * W,
                                          keep=[self.arena])
        self.slot_table = T.PointerTable(list(bases), [W * Ns] * W, keep=[self.arena])
        with _LOCK:
            _AG[self.arena.data_ptr()] = self
            _RS[self.rs_input.data_ptr()] = self
        self.placements = 0
        self.reductions = 0
        # plans for the parameters that get gradients, when some do not (frozen ones): FSDP2
        # reduce-scatters only those, in group order, so their shapes fix the layout
        self._sub_plans = {}
        self.pending = None   # (one-rank plan, shard numel, fp32?) of the staged reduction
        # fp32 slots for gradients FSDP2 accumulated with sync off (made on first use)
        self.arena32 = None
        self.peers32 = None
        self.slot_table32 = None

    def ensure_arena32(self) -> None:
        """This rank's fp32 [W][Ns] slot, mapped into every rank (a collective on first use:
        every rank stages fp32 gradients at the same backward)."""
        import torch
        if self.arena32 is not None:
            return
        W, Ns = self.world, self.shard_numel
        arena32 = torch.zeros(W * Ns, dtype=torch.float32, device=self.device)
        torch.cuda.synchronize(self.device)
        exports = X.all_exports(X.export({"arena32": arena32}), self.group)
        self.peers32 = X.PeerMaps(exports, self.rank, self.device.index,
                                  {"arena32": arena32.data_ptr()})
        self.slot_table32 = T.PointerTable(list(self.peers32.bases("arena32", W)), [W * Ns] * W,
                                           keep=[arena32])
        self.arena32 = arena32

    def plans_for(self, shapes):
        """(all-rank plan, one-rank plan, shard numel) for a reduction over `shapes`."""
        shapes = tuple(tuple(int(d) for d in s) for s in shapes)
        if list(shapes) == self.shapes:
            return self.plan, self.rank_plan, self.shard_numel
        ent = self._sub_plans.get(shapes)
        if ent is None:
            plan = T.Plan(shapes, self.world, device=self.device)
            ent = (plan, T.Plan(shapes, self.world, device=self.device, rank=self.rank),
                   plan.shard_numel)
            self._sub_plans[shapes] = ent
        return ent

    def meet(self, device_wide: bool = False) -> None:
        """Wait for this rank's work on the current stream (where FSDP2 issues the collective,
        after its copy-in or pack; and where this group enqueued its placement or reduction),
        then meet every rank.  Work that FSDP2 queued on other streams, compute among it, keeps
        running.  device_wide: wait for every stream of the device instead."""
        import torch
        import torch.distributed as dist
        if device_wide:
            torch.cuda.synchronize(self.device)
        else:
            torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(self.group)

    def place(self, out) -> None:
        """FSDP2's copy-out: every rank's row into the unsharded parameters (TIDE-AG)."""
        if len(out) != len(self.shapes):
            raise ValueError("copy-out outputs do not match the group's parameters")
        for t, c in zip(out, self.chunks):
            if t.numel() != self.world * c or not t.is_contiguous():
                raise ValueError("copy-out output is not a parameter's padded storage")
        self.plan.ag_gather_place(self.shard_table, T.TensorTable(list(out)), engine=self.engine)
        self.meet()                                   # every rank has read every row
        self.placements += 1

    def stage(self, grads) -> None:
        """FSDP2's pack: this rank's bf16 gradients into its arena (Slot-Reuse phase 1).  The
        gradients are those of the group's parameters that got one, in group order."""
        f32 = _check_grads(grads, len(self.shapes))
        plan, rank_plan, ns = self.plans_for([tuple(g.shape) for g in grads])
        if f32:
            self.ensure_arena32()
            plan.rs_stage_one_f32(T.TensorTable(list(grads)), self.arena32, engine=self.engine)
        else:
            plan.rs_stage_one(T.TensorTable(list(grads)), self.arena, engine=self.engine)
        self.pending = (rank_plan, ns, f32)

    def reduce(self, out, op) -> None:
        """The reduce-scatter: this rank's fp32 shard from rows r of every arena (TIDE-RS)."""
        import torch
        import torch.distributed as dist
        if self.pending is None:
            raise ValueError("reduce-scatter without staged gradients")
        rank_plan, ns, f32 = self.pending
        self.pending = None
        if out.dtype != torch.float32 or out.numel() != ns or not out.is_contiguous():
            raise ValueError("reduce-scatter output is not this rank's fp32 shard")
        if op == dist.ReduceOp.AVG:
            scale = T.TIDE_SCALE_INV_WORLD
        elif op == dist.ReduceOp.SUM:
            scale = T.TIDE_SCALE_NONE
        else:
            raise ValueError(f"reduce op {op} is not a sum or an average")
        self.meet()                                   # every rank's gradients are staged
        if f32:
            rank_plan.rs_reduce_slots_f32(self.slot_table32, out, scale_mode=scale)
        else:
            rank_plan.rs_reduce_slots(self.slot_table, out, scale_mode=scale, order=self.order)
        self.meet()                                   # nobody copies in over a row still read
        self.reductions += 1

    def close(self) -> None:
        """Unmap the peers' arenas once no rank can still read them (a collective)."""
        if self.peers is None:
            return
        self.meet(device_wide=True)
        with _LOCK:
            _AG.pop(self.arena.data_ptr(), None)
            _RS.pop(self.rs_input.data_ptr(), None)
        self.peers.close()
        if self.peers32 is not None:
            self.peers32.close()
            self.peers32 = None
        self.meet(device_wide=True)
        self.peers = None


def _comm_classes():
    from torch.distributed.fsdp._fully_shard._fsdp_api import AllGather, ReduceScatter

    class TideAllGather(AllGather):
        """FSDP2's all-gather for a TIDE group: the buffer is the group's arena; the call
        waits for every rank's row (the placement runs in FSDP2's copy-out)."""

        def __init__(self, tg: TideGroup):
            self.tg = tg

        def allocate(self, size, *, dtype, device):
            import torch
            if dtype != torch.bfloat16 or math.prod(int(s) for s in size) != self.tg.arena.numel():
                raise ValueError("all-gather buffer is not the group's bf16 [W][Ns] arena")
            return self.tg.arena

        def __call__(self, output_tensor, input_tensor, group, async_op=False):
            if output_tensor.data_ptr() != self.tg.arena.data_ptr():
                raise ValueError("all-gather output is not the group's arena")
            self.tg.meet()                            # every rank's row is in its arena
            return None

    class TideReduceScatter(ReduceScatter):
        """FSDP2's reduce-scatter for a TIDE group: no fp32 input buffer; the reduction
        reads every rank's staged arena."""

        def __init__(self, tg: TideGroup):
            self.tg = tg

        def allocate(self, size, *, dtype, device):
            # FSDP2 asks for the packed input, packs (the staging), then asks for the output
            import torch
            n = math.prod(int(s) for s in size)
            if dtype != torch.float32:
                raise ValueError("TIDE's reduce-scatter reduces into fp32")
            if self.tg.pending is None:
                if n % self.tg.world or n > self.tg.world * self.tg.shard_numel:
                    raise ValueError("unexpected reduce-scatter input size")
                return self.tg.rs_input.expand(n)     # FSDP2's packed input: never materialized
            if n != self.tg.pending[1]:
                raise ValueError("unexpected reduce-scatter output size")
            return torch.empty(n, dtype=torch.float32, device=self.tg.device)

        def __call__(self, output_tensor, input_tensor, group, op, async_op=False):
            if input_tensor.data_ptr() != self.tg.rs_input.data_ptr():
                raise ValueError("reduce-scatter input is not the group's")
            self.tg.reduce(output_tensor, op)
            return None

    return TideAllGather, TideReduceScatter


def _install(dispatch_key: str = "CUDA") -> None:
    """Route FSDP2's copy-out and pack on `dispatch_key` tensors to the registered groups
    (_AG, _RS); every other buffer keeps FSDP2's own implementation."""
    if dispatch_key in _INSTALLED:
        return
    import torch
    from torch.distributed.fsdp._fully_shard import _fsdp_collectives as C

    stock_split, stock_cat = C.split_with_sizes_copy, C.chunk_cat

    def split_with_sizes_copy(all_gather_output, all_gather_input_split_sizes, dim=0, *, out):
        tg = _AG.get(all_gather_output.data_ptr())
        if tg is None:
            return stock_split(all_gather_output, all_gather_input_split_sizes, dim, out=out)
        if dim != 1 or list(all_gather_input_split_sizes) != tg.chunks:
            raise ValueError("copy-out of a TIDE group with another layout")
        tg.place(out)

    def chunk_cat(tensors, dim, num_chunks, out):
        tg = _RS.get(out.data_ptr())
        if tg is None:
            return stock_cat(tensors, dim, num_chunks, out)
        if dim != 0 or num_chunks != tg.world:
            raise ValueError("pack of a TIDE group with another layout")
        tg.stage(tensors)

    lib = torch.library.Library("fsdp", "IMPL")  # noqa: TOR901
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")           # replacing FSDP2's kernels is the point
        lib.impl("split_with_sizes_copy", split_with_sizes_copy, dispatch_key, allow_override=True)
        lib.impl("chunk_cat", chunk_cat, dispatch_key, allow_override=True)
    _LIBS.append(lib)                             # the registrations live as long as the library
    _INSTALLED.add(dispatch_key)


def fully_shard_tide(module, group=None, *, reshard_after_forward=None,
                     engine: int = T.TIDE_ENGINE_SM, order: int = T.TIDE_ORDER_RANK):
    """``fully_shard(module)`` over `group` with bf16 compute parameters and fp32 gradient
    reduction, its all-gather and reduce-scatter done by TIDE.  Apply it to submodules
    first, then to the root, in the same order on every rank.  Returns the module.

    reshard_after_forward: as FSDP2's (None: True for submodules, False for the root), except
    that resharding to a smaller world (an int) is refused: every all-gather of a TIDE group
    spans the whole group."""
    import torch
    import torch.distributed as dist
    from torch.distributed.device_mesh import DeviceMesh
    from torch.distributed.fsdp import MixedPrecisionPolicy, fully_shard

    if not (reshard_after_forward is None or isinstance(reshard_after_forward, bool)):
        raise ValueError("TIDE groups reshard to the whole group or not at all")
    _install()
    pg = group if group is not None else dist.group.WORLD
    mesh = DeviceMesh.from_group(pg, "cuda")
    fully_shard(module, mesh=mesh, reshard_after_forward=reshard_after_forward,
                mp_policy=MixedPrecisionPolicy(param_dtype=torch.bfloat16, reduce_dtype=torch.float32))
    param_group = module._get_fsdp_state()._fsdp_param_group
    if param_group is None:                       # every parameter belongs to a submodule
        return module
    shapes = [tuple(fp._orig_size) for fp in param_group.fsdp_params]
    tg = TideGroup(shapes, pg, engine=engine, order=order)
    ag_cls, rs_cls = _comm_classes()
    module.set_custom_all_gather(ag_cls(tg))
    module.set_custom_reduce_scatter(rs_cls(tg))
    module._tide_group = tg
    return module


def tide_groups(module) -> list:
    """The TIDE groups of `module` and its submodules, in module order."""
    return [m._tide_group for m in module.modules() if getattr(m, "_tide_group", None) is not None]


def close(module) -> None:
    """Unmap every TIDE group of `module` (a collective: all ranks, same order)."""
    for tg in tide_groups(module):
        tg.close()
