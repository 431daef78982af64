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


def fsdp2_tide_worker(rank, world, port, steps, lr, out_dir, engine, order):
    import torch
    import torch.distributed as dist
    from fsdp2_layout_aware_b200 import fsdp2 as F
    from _gpu_helpers import bits_of

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        torch.manual_seed(0)                      # the same initial parameters on every rank
        model = _net().cuda()
        for m in (model.l1, model.l2, model):
            F.fully_shard_tide(m, engine=engine, order=order)
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
            for i, t in enumerate(grads):
                save(f"grad_{g}_{n}_{rank}_{i}.npy", bits_of(t))
            save(f"slot0_{g}_{n}_{rank}.npy", bits_of(tg.arena))
            stage0(tg, grads)
            torch.cuda.synchronize()
            save(f"slot1_{g}_{n}_{rank}.npy", bits_of(tg.arena))

        def reduce(tg, out, op):
            g, n = tick("reduce", tg)
            reduce0(tg, out, op)
            save(f"shard_{g}_{n}_{rank}.npy", out.cpu().numpy())

        F.TideGroup.place, F.TideGroup.stage, F.TideGroup.reduce = place, stage, reduce
        opt = torch.optim.SGD(model.parameters(), lr=lr)
        gen = torch.Generator(device="cuda").manual_seed(100 + rank)
        x = torch.randn(16, 40, device="cuda", generator=gen)
        y = torch.randn(16, 10, device="cuda", generator=gen)
        losses = []
        for _ in range(steps):
            loss = ((model(x).float() - y) ** 2).mean()
            loss.backward()
            opt.step()
            opt.zero_grad()
            losses.append(float(loss))
        with open(os.path.join(out_dir, f"counts_{rank}.json"), "w") as f:
            json.dump({f"{k[0]}_{k[1]}": v for k, v in count.items()} | {"losses": losses}, f)
        F.close(model)
    finally:
        dist.destroy_process_group()
