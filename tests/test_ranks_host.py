"""One-rank plans across processes (gloo on CPU, no GPU): each rank builds only its own
plan, and the ranks' tile lists together are the all-rank plan's, shifted into each
rank's shard."""
import datetime
import os

import pytest
import torch.multiprocessing as mp

from _dist_helpers import free_port

SHAPES = ((37, 16), (1000,), (7, 3), (5, 130), (0, 4), (64, 64))


def _worker(rank, world, port, out_dir):
    import json

    import torch.distributed as dist

    from fsdp2_layout_aware_b200 import tide as T
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        plan = T.Plan(SHAPES, world, host_only=True, rank=rank)
        mine = [(t.src_off, t.dst_off, t.param, t.rank, t.n_valid, t.n_total) for t in plan.tiles()]
        gathered = [None] * world
        dist.all_gather_object(gathered, (plan.shard_numel, mine))
        if rank == 0:
            with open(os.path.join(out_dir, "tiles.json"), "w") as f:
                json.dump(gathered, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_rank_plans_across_processes_make_up_the_group(world, tmp_path):
    import json

    from fsdp2_layout_aware_b200 import tide as T
    mp.spawn(_worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    gathered = json.load(open(tmp_path / "tiles.json"))
    full = T.Plan(SHAPES, world, host_only=True)
    Ns = full.shard_numel
    assert all(ns == Ns for ns, _ in gathered)
    union = sorted((s, d + r * Ns, p, rk, v, n) for r, (_, tiles) in enumerate(gathered)
                   for (s, d, p, rk, v, n) in tiles)
    ref = sorted((t.src_off, t.dst_off, t.param, t.rank, t.n_valid, t.n_total) for t in full.tiles())
    assert union == ref
    for r, (_, tiles) in enumerate(gathered):
        assert all(rk == r and 0 <= d and d + n <= Ns for (_, d, _, rk, _, n) in tiles)

