"""Process body for the sharded-data-parallel test: n processes share one GPU, each a rank of
a small bf16 network trained with fsdp2_layout_aware_b200.fsdp.ShardedParams; each saves what the
test checks against the oracle (its gradients, its reduced gradient shard, its shard and the
parameters placed from every rank's shards)."""
import datetime
import os

import numpy as np


def _net():
    import torch

    class Net(torch.nn.Module):
        """Two linear layers and a (1, 10) output scale: its one row leaves every rank but
        rank 0 a shard of pad rows only."""

        def __init__(self):
            super().__init__()
            self.scale = torch.nn.Parameter(torch.linspace(0.5, 1.5, 10).reshape(1, 10))
            self.l1 = torch.nn.Linear(40, 24)
            self.l2 = torch.nn.Linear(24, 10)

        def forward(self, x):
            return self.l2(torch.relu(self.l1(x))) * self.scale

    return Net()


def train_worker(rank, world, port, steps, lr, out_dir, shapes):
    import torch
    import torch.distributed as dist
    from fsdp2_layout_aware_b200.fsdp import ShardedParams
    from _gpu_helpers import bits_of

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        torch.manual_seed(0)                      # the same initial parameters on every rank
        model = _net().to(device="cuda", dtype=torch.bfloat16)
        params = list(model.parameters())
        assert [tuple(p.shape) for p in params] == [tuple(s) for s in shapes]
        sp = ShardedParams(params)
        gen = torch.Generator(device="cuda").manual_seed(100 + rank)
        x = torch.randn(16, 40, device="cuda", dtype=torch.bfloat16, generator=gen)
        y = torch.randn(16, 10, device="cuda", dtype=torch.bfloat16, generator=gen)
        for step in range(steps):
            sp.unshard()
            torch.cuda.synchronize()
            for i, p in enumerate(params):
                np.save(os.path.join(out_dir, f"placed_{step}_{rank}_{i}.npy"), bits_of(sp.storage[i]))
            sp.zero_grad()
            loss = ((model(x).float() - y.float()) ** 2).mean()
            loss.backward()
            torch.cuda.synchronize()
            for i, p in enumerate(params):
                assert p.grad.data_ptr() == sp.grad_arena.data_ptr() + 2 * sp.layout.grad_off[i]
                np.save(os.path.join(out_dir, f"grad_{step}_{rank}_{i}.npy"), bits_of(p.grad))
            sp.reduce_grads()
            torch.cuda.synchronize()
            np.save(os.path.join(out_dir, f"gshard_{step}_{rank}.npy"), sp.grad_shard.cpu().numpy())
            np.save(os.path.join(out_dir, f"master0_{step}_{rank}.npy"), sp.master.cpu().numpy())
            sp.sgd_step(lr)
            torch.cuda.synchronize()
            np.save(os.path.join(out_dir, f"master1_{step}_{rank}.npy"), sp.master.cpu().numpy())
            np.save(os.path.join(out_dir, f"shard_{step}_{rank}.npy"), bits_of(sp.shard))
        sp.close()
    finally:
        dist.destroy_process_group()
