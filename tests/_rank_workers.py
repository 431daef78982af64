"""Rank processes for the multi-process tests: W processes share one GPU, each owning its own
gradients and its own all-gather shard, and reach each other's through CUDA IPC.  The IPC
mappings enter the pointer tables the way peer-mapped memory of other GPUs would."""
import datetime
import os

import numpy as np


def rank_worker(rank, world, port, shapes, seed, queues, out_dir):
    import torch
    import torch.distributed as dist

    import synth
    from fsdp2_layout_aware_b200 import tide as T
    from synth import configs
    from _gpu_helpers import bits_of, to_dev

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        group = configs.Group("ranks", world, tuple(shapes))
        full = T.Plan(group.shapes, world)
        Ns = full.shard_numel
        # this rank's own data: its gradients and its shard of the all-gather input
        own = [to_dev(synth.grad_host(group, seed, rank, i), group.shapes[i])
               for i in range(group.n_params)]
        shard = to_dev(synth.ag_host(group, Ns, seed).reshape(world, Ns)[rank])
        torch.cuda.synchronize()
        for r in range(world):
            if r != rank:
                queues[r].put((rank, own, shard))
        grads, shards = [None] * world, [None] * world
        grads[rank], shards[rank] = own, shard
        for _ in range(world - 1):
            k, g, s = queues[rank].get(timeout=120)
            grads[k], shards[k] = g, s
        dist.barrier()                       # every rank's data is in place
        # TIDE-RS: this rank reduces its own shard from every rank's gradients
        mine = T.Plan(group.shapes, world, rank=rank)
        out = torch.full((Ns,), float("nan"), device="cuda")
        mine.rs_reduce(grads, out, scale_mode=T.TIDE_SCALE_INV_WORLD)
        tree = torch.full((Ns,), float("nan"), device="cuda")
        mine.rs_reduce(grads, tree, scale_mode=T.TIDE_SCALE_NONE, order=T.TIDE_ORDER_TREE)
        # TIDE-AG: every rank's shard placed into this rank's parameter storage
        placed = {}
        for engine, name in ((T.TIDE_ENGINE_SM, "sm"), (T.TIDE_ENGINE_CE, "ce")):
            params = [torch.full((full.query(i)["padded_numel"],), 0x7777, dtype=torch.int16,
                                 device="cuda").view(torch.bfloat16) for i in range(group.n_params)]
            full.ag_gather_place(shards, params, engine=engine)
            placed[name] = params
        torch.cuda.synchronize()
        mine.check()
        full.check()
        np.save(os.path.join(out_dir, f"rs_{rank}.npy"), out.cpu().numpy())
        np.save(os.path.join(out_dir, f"tree_{rank}.npy"), tree.cpu().numpy())
        for name, params in placed.items():
            for i, p in enumerate(params):
                np.save(os.path.join(out_dir, f"ag_{name}_{rank}_{i}.npy"), bits_of(p))
        del grads, shards, g, s
        torch.cuda.synchronize()
        dist.barrier()                       # no rank frees its buffers while a peer may read them
    finally:
        dist.destroy_process_group()
