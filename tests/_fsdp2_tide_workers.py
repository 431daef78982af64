"""Process body for the FSDP2 test: n processes share one GPU, each a rank of FSDP2's own
fully_shard with TIDE's collectives (fsdp2_layout_aware_b200.fsdp2).  The TIDE group's
placement, staging and reduction are wrapped in this process only, to save what the test
checks against the oracle: each rank's all-gather row and the parameters it placed, its
gradients and its arena before and after staging, and its reduced fp32 shard."""
import collections
import datetime
import json
import os

import numpy as np


def _net():
    import torch

    class Net(torch.nn.Module):
        """Two linear layers and a (1, 10) output scale, the root's own parameter: its one
        row leaves every rank but rank 0 a shard of pad rows only."""

        def __init__(self):
            super().__init__()
            self.scale = torch.nn.Parameter(torch.linspace(0.5, 1.5, 10).reshape(1, 10))
            self.l1 = torch.nn.Linear(40, 24)
            self.l2 = torch.nn.Linear(24, 10)

        def forward(self, x):
            return self.l2(torch.relu(self.l1(x))) * self.scale

    return Net()


MODES = ("plain", "frozen", "accum", "no_reshard", "accum_unsynced")


def _backward(model, x, y, mode):
    """One step's backward on (x, y).  accum: two micro-batches, each reduce-scattered (FSDP2
    sums the fp32 shards); accum_unsynced: the first with FSDP2's gradient sync off (its
    unsharded gradients kept, in fp32, for the second).  Returns the last loss."""
    if mode in ("accum", "accum_unsynced"):
        model.set_requires_gradient_sync(mode == "accum")
        ((model(x[:8]).float() - y[:8]) ** 2).mean().backward()
        model.set_requires_gradient_sync(True)
        loss = ((model(x[8:]).float() - y[8:]) ** 2).mean()
    else:
        loss = ((model(x).float() - y) ** 2).mean()
    loss.backward()
    return float(loss)


def _train(model, opt, x, y, steps, mode):
    losses = []
    for _ in range(steps):
        losses.append(_backward(model, x, y, mode))
        opt.step()
        opt.zero_grad()
    return losses


def _shard_args(mode):
    """fully_shard keyword arguments of a test mode (FSDP2's default otherwise: resharded
    after forward, the root excepted)."""
    return {"reshard_after_forward": False} if mode == "no_reshard" else {}


def fsdp2_tide_worker(rank, world, port, steps, lr, out_dir, engine, order, mode="plain"):
    import torch
    import torch.distributed as dist
    from fsdp2_layout_aware_b200 import fsdp2 as F
    from _gpu_helpers import bits_of, f32_bits

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        torch.manual_seed(0)                      # the same initial parameters on every rank
        model = _net().cuda()
        if mode == "frozen":
            model.l1.bias.requires_grad_(False)      # left out of its group's reduce-scatter
        for m in (model.l1, model.l2, model):
            F.fully_shard_tide(m, engine=engine, order=order, **_shard_args(mode))
        groups = F.tide_groups(model)
        gid = {id(tg): g for g, tg in enumerate(groups)}
        if rank == 0:
            with open(os.path.join(out_dir, "shapes.json"), "w") as f:
                json.dump([tg.shapes for tg in groups], f)
        count = collections.Counter()
        place0, stage0, reduce0 = F.TideGroup.place, F.TideGroup.stage, F.TideGroup.reduce

        def save(name, arr):
            np.save(os.path.join(out_dir, name), arr)

        def tick(kind, tg):
            g = gid[id(tg)]
            n = count[(kind, g)]
            count[(kind, g)] += 1
            return g, n

        def place(tg, out):
            g, n = tick("place", tg)
            torch.cuda.synchronize()
            Ns = tg.shard_numel
            save(f"row_{g}_{n}_{rank}.npy", bits_of(tg.arena[rank * Ns:(rank + 1) * Ns]))
            place0(tg, out)
            for i, t in enumerate(out):
                save(f"placed_{g}_{n}_{rank}_{i}.npy", bits_of(t))

        def stage(tg, grads):
            g, n = tick("stage", tg)
            torch.cuda.synchronize()
            f32 = grads[0].dtype == torch.float32    # accumulated with gradient sync off
            if rank == 0:
                with open(os.path.join(out_dir, f"staged_shapes_{g}_{n}.json"), "w") as f:
                    json.dump({"shapes": [tuple(t.shape) for t in grads], "f32": f32}, f)
            bits = f32_bits if f32 else bits_of
            for i, t in enumerate(grads):
                save(f"grad_{g}_{n}_{rank}_{i}.npy", bits(t))
            if f32:
                tg.ensure_arena32()
            arena = (lambda: tg.arena32) if f32 else (lambda: tg.arena)
            save(f"slot0_{g}_{n}_{rank}.npy", bits(arena()))
            stage0(tg, grads)
            torch.cuda.synchronize()
            save(f"slot1_{g}_{n}_{rank}.npy", bits(arena()))

        def reduce(tg, out, op):
            g, n = tick("reduce", tg)
            reduce0(tg, out, op)
            save(f"shard_{g}_{n}_{rank}.npy", out.cpu().numpy())

        F.TideGroup.place, F.TideGroup.stage, F.TideGroup.reduce = place, stage, reduce
        opt = torch.optim.SGD(model.parameters(), lr=lr)
        gen = torch.Generator(device="cuda").manual_seed(100 + rank)
        x = torch.randn(16, 40, device="cuda", generator=gen)
        y = torch.randn(16, 10, device="cuda", generator=gen)
        losses = _train(model, opt, x, y, steps, mode)
        with open(os.path.join(out_dir, f"counts_{rank}.json"), "w") as f:
            json.dump({f"{k[0]}_{k[1]}": v for k, v in count.items()} | {"losses": losses}, f)
        F.close(model)
    finally:
        dist.destroy_process_group()


class OracleGroup:
    """A TIDE group for FSDP2 on the CPU whose placement, staging and reduction are the
    oracle's, with gloo collectives standing in for the peer reads: it checks FSDP2's side of
    fsdp2_layout_aware_b200.fsdp2 (which buffers it asks for, in which order, and what lands
    where) without a GPU."""

    def __init__(self, shapes):
        import torch
        import torch.distributed as dist
        from fsdp2_layout_aware_b200 import fsdp2 as F
        from fsdp2_layout_aware_b200 import tide as T
        self.world, self.rank = dist.get_world_size(), dist.get_rank()
        self.shapes = [tuple(int(d) for d in s) for s in shapes]
        plan = T.Plan(self.shapes, self.world, host_only=True)
        self.shard_numel = plan.shard_numel
        self.chunks = [plan.query(i)["chunk_numel"] for i in range(len(self.shapes))]
        self.arena = torch.zeros(self.world * self.shard_numel, dtype=torch.bfloat16)
        self.rs_input = torch.zeros(1)
        self.device = torch.device("cpu")
        self.calls = []
        self.pending = None
        self.arena32 = None
        F._AG[self.arena.data_ptr()] = self
        F._RS[self.rs_input.data_ptr()] = self

    def meet(self):
        import torch.distributed as dist
        dist.barrier()

    def _all(self, t):
        import torch
        import torch.distributed as dist
        bufs = [torch.empty_like(t) for _ in range(self.world)]
        dist.all_gather(bufs, t.contiguous())
        return [b.view(torch.int16).numpy().view(np.uint16) for b in bufs]

    def _all32(self, t):
        import torch
        import torch.distributed as dist
        bufs = [torch.empty_like(t) for _ in range(self.world)]
        dist.all_gather(bufs, t.contiguous())
        return [b.numpy() for b in bufs]

    def place(self, out):
        import oracle
        import torch
        self.calls.append("place")
        Ns, r = self.shard_numel, self.rank
        rows = self._all(self.arena[r * Ns:(r + 1) * Ns])
        want = oracle.ag_copyout(self.world, self.shapes, np.concatenate(rows))
        for t, w in zip(out, want):
            t.view(-1).view(torch.int16).copy_(torch.from_numpy(w.view(np.int16)))
        self.meet()

    def stage(self, grads):
        import oracle
        import torch
        from fsdp2_layout_aware_b200 import fsdp2 as F
        f32 = F._check_grads(grads, len(self.shapes))
        self.calls.append("stage")
        shapes = [tuple(g.shape) for g in grads]            # the parameters that got gradients
        ns = oracle.layout(self.world, shapes).Ns
        if f32:                                             # accumulated with gradient sync off
            if self.arena32 is None:
                self.arena32 = torch.zeros(self.world * self.shard_numel)
            words = [g.detach().contiguous().numpy().reshape(-1).view(np.uint32) for g in grads]
            slot = self.arena32.numpy().view(np.uint32)     # shares the fp32 slot's memory
            oracle.slot_stage_f32(self.world, shapes, words, slot[:self.world * ns])
        else:
            bits = [g.detach().contiguous().view(torch.int16).numpy().reshape(-1).view(np.uint16)
                    for g in grads]
            slot = self.arena.view(torch.int16).numpy().view(np.uint16)   # shares the arena's memory
            oracle.slot_stage(self.world, shapes, bits, slot[:self.world * ns])
        self.pending = (shapes, ns, f32)

    def reduce(self, out, op):
        import oracle
        import torch
        import torch.distributed as dist
        self.calls.append("reduce")
        shapes, ns, f32 = self.pending
        self.pending = None
        self.meet()
        scale = 1 if op == dist.ReduceOp.AVG else 0
        if f32:
            slots = [s[:self.world * ns] for s in self._all32(self.arena32)]
            res = oracle.rs_reduce_slots_f32(self.world, shapes, slots, scale)
        else:
            slots = [s[:self.world * ns] for s in self._all(self.arena)]
            res = oracle.rs_reduce_slots(self.world, shapes, slots, scale)
        r = self.rank
        out.copy_(torch.from_numpy(res[r * ns:(r + 1) * ns].copy()))
        self.meet()


def fsdp2_oracle_worker(rank, world, port, steps, lr, out_dir, mode="plain"):
    """Stock FSDP2, then FSDP2 with the TIDE comms and operator routing of
    fsdp2_layout_aware_b200.fsdp2 over OracleGroups, on the CPU; saves both runs' sharded
    gradients of every step and final sharded parameters."""
    import torch
    import torch.distributed as dist
    from torch.distributed.device_mesh import DeviceMesh
    from torch.distributed.fsdp import MixedPrecisionPolicy, fully_shard
    from fsdp2_layout_aware_b200 import fsdp2 as F

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        mesh = DeviceMesh.from_group(dist.group.WORLD, "cpu")
        policy = MixedPrecisionPolicy(param_dtype=torch.bfloat16, reduce_dtype=torch.float32)
        gen = torch.Generator().manual_seed(100 + rank)
        x, y = torch.randn(16, 40, generator=gen), torch.randn(16, 10, generator=gen)
        calls = {}
        for arm in ("stock", "tide"):
            torch.manual_seed(0)
            model = _net()
            if mode == "frozen":
                model.l1.bias.requires_grad_(False)   # left out of its group's reduce-scatter
            groups = []
            for m in (model.l1, model.l2, model):
                fully_shard(m, mesh=mesh, mp_policy=policy, **_shard_args(mode))
                if arm == "tide":
                    F._install("CPU")
                    pg = m._get_fsdp_state()._fsdp_param_group
                    tg = OracleGroup([tuple(fp._orig_size) for fp in pg.fsdp_params])
                    ag_cls, rs_cls = F._comm_classes()
                    m.set_custom_all_gather(ag_cls(tg))
                    m.set_custom_reduce_scatter(rs_cls(tg))
                    groups.append(tg)
            opt = torch.optim.SGD(model.parameters(), lr=lr)
            for step in range(steps):
                _backward(model, x, y, mode)
                for i, p in enumerate(model.parameters()):
                    if p.grad is not None:
                        np.save(os.path.join(out_dir, f"{arm}_grad_{step}_{rank}_{i}.npy"),
                                p.grad.to_local().detach().numpy())
                opt.step()
                opt.zero_grad()
            for i, p in enumerate(model.parameters()):
                np.save(os.path.join(out_dir, f"{arm}_param_{rank}_{i}.npy"), p.to_local().detach().numpy())
            calls[arm] = [tg.calls for tg in groups]
        with open(os.path.join(out_dir, f"calls_{rank}.json"), "w") as f:
            json.dump(calls["tide"], f)
    finally:
        dist.destroy_process_group()
