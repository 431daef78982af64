"""Multi-process helpers (gloo on CPU) used by the tests."""
import os
import socket

import numpy as np


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rs_worker(rank, world, port, in_dir):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        buf = torch.from_numpy(np.load(os.path.join(in_dir, f"packed_{rank}.npy")))
        shard = torch.empty(buf.numel() // world, dtype=buf.dtype)
        dist.reduce_scatter_tensor(shard, buf, op=dist.ReduceOp.SUM)
        np.save(os.path.join(in_dir, f"shard_{rank}.npy"), shard.numpy())
    finally:
        dist.destroy_process_group()


def run_gloo_reduce_scatter(packed, tmp_dir):
    """Each of W processes contributes packed[k] (fp32 [W*Ns]); returns the W shards."""
    import torch.multiprocessing as mp
    world = len(packed)
    for k, p in enumerate(packed):
        np.save(os.path.join(tmp_dir, f"packed_{k}.npy"), p)
    mp.spawn(_rs_worker, args=(world, free_port(), str(tmp_dir)), nprocs=world, join=True)
    return [np.load(os.path.join(tmp_dir, f"shard_{k}.npy")) for k in range(world)]


def run_procs(target, n, args):
    """Run target(p, *args(port)) in n spawned processes (p = 0..n-1) and require each to exit
    0 within 300 s."""
    import torch
    ctx = torch.multiprocessing.get_context("spawn")
    port = free_port()
    procs = [ctx.Process(target=target, args=(p, *args(port))) for p in range(n)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.terminate()
        p.join(timeout=30)
    assert not alive, "a process did not finish"
    assert [p.exitcode for p in procs] == [0] * n
