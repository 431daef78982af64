"""One-rank plans and placement from per-rank shards: the data-parallel exchange as each rank
runs it.

Rank r reduces only its own shard, reading chunk r of every rank's gradients through the
pointer table; it places every rank's shard into its parameters, reading each shard where it
lies.  On one GPU the ranks are either W plans in one process (separate buffers) or W
processes that share their buffers through CUDA IPC.  No kernel waits on another: the
processes meet only at host barriers, before and after the calls.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from fsdp2_layout_aware_b200 import tide as T
from synth import configs

from _dist_helpers import free_port
from _gpu_helpers import bits_of, f32_bits, grads_to_dev, to_dev
from _groups import degenerate, mini_sweep, mini_wan

pytestmark = pytest.mark.gpu

GROUPS = [configs.tiny(), degenerate(), mini_wan(), configs.qwen3moe(4), mini_sweep(8),
          configs.Group("ragged_w3", 3, ((37, 16), (1000,), (7, 3), (5, 130)))]
IDS = [f"{g.name}_w{g.world}" for g in GROUPS]


@pytest.mark.parametrize("group", GROUPS, ids=IDS)
def test_rank_plans_reduce_their_own_shards(group):
    W = group.world
    grads = synth.grads_host(group, seed=71)
    dev = grads_to_dev(group, grads)
    L = oracle.layout(W, group.shapes)
    ref = oracle.rs_reduce(W, group.shapes, grads, 1).view(np.uint32).reshape(W, L.Ns)
    tree = oracle.rs_reduce_tree(W, group.shapes, grads, 0).view(np.uint32).reshape(W, L.Ns)
    full = T.Plan(group.shapes, W)
    for r in range(W):
        plan = T.Plan(group.shapes, W, rank=r)
        out = torch.full((L.Ns,), float("nan"), device="cuda")
        plan.rs_reduce(dev, out, scale_mode=T.TIDE_SCALE_INV_WORLD)
        torch.cuda.synchronize()
        plan.check()
        assert np.array_equal(f32_bits(out), ref[r])
        if plan.n_tiles:
            k, n = plan.last_launch()
            assert k in (T.K_RS, T.K_RS_V32) and n == plan.launch_ctas(k, 0)
        plan.rs_reduce(dev, out, scale_mode=T.TIDE_SCALE_NONE, order=T.TIDE_ORDER_TREE)
        torch.cuda.synchronize()
        assert np.array_equal(f32_bits(out), tree[r])
        tma = T.Plan(group.shapes, W, rank=r, tma=True)
        out.fill_(float("nan"))
        tma.rs_reduce(dev, out, scale_mode=T.TIDE_SCALE_INV_WORLD)
        torch.cuda.synchronize()
        assert np.array_equal(f32_bits(out), ref[r])
    assert sum(T.Plan(group.shapes, W, rank=r).n_tiles for r in range(W)) == full.n_tiles


@pytest.mark.parametrize("group", GROUPS, ids=IDS)
@pytest.mark.parametrize("engine", [T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE], ids=["sm", "ce"])
def test_gather_place_from_separate_shards(group, engine):
    W = group.world
    L = oracle.layout(W, group.shapes)
    plan = T.Plan(group.shapes, W)
    ag = synth.ag_host(group, L.Ns, seed=72).reshape(-1)
    ref = oracle.ag_copyout(W, group.shapes, ag)
    # each rank's shard is its own buffer, with its pad positions poisoned (never read)
    rows = ag.reshape(W, L.Ns).copy()
    for i in range(group.n_params):
        for r in range(W):
            valid = max(0, min(L.c[i], group.numel(i) - r * L.c[i]))
            rows[r, L.off[i] + valid: L.off[i] + L.c[i]] = 0xFFFF
    shards = [to_dev(rows[r]) for r in range(W)]
    params = [torch.full((plan.query(i)["padded_numel"],), 0x7777, dtype=torch.int16,
                         device="cuda").view(torch.bfloat16) for i in range(group.n_params)]
    plan.ag_gather_place(shards, params, engine=engine)
    torch.cuda.synchronize()
    plan.check()
    for p, r in zip(params, ref):
        assert np.array_equal(bits_of(p), r)
    if plan.n_tiles:
        k, n = plan.last_launch()
        assert (k, n) == ((T.K_AG_GATHER, plan.launch_ctas(T.K_AG_GATHER, 0))
                          if engine == T.TIDE_ENGINE_SM else (-1, 0))


@pytest.mark.parametrize("world", [2, 4])
def test_ranks_as_processes_through_cuda_ipc(world, tmp_path):
    """W processes on one GPU, each holding only its own gradients and shard: each reduces its
    own shard and places all shards, reading the peers' buffers through CUDA IPC."""
    from _rank_workers import rank_worker
    shapes = ((37, 16), (1000,), (7, 3), (5, 130), (64, 64), (8 * world + 3, 40))
    seed = 73
    ctx = torch.multiprocessing.get_context("spawn")
    queues = [ctx.Queue() for _ in range(world)]
    port = free_port()
    procs = [ctx.Process(target=rank_worker,
                         args=(r, world, port, shapes, seed, queues, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.terminate()
        p.join(timeout=30)
    assert not alive, "a rank process did not finish"
    assert [p.exitcode for p in procs] == [0] * world
    group = configs.Group("ranks", world, shapes)
    L = oracle.layout(world, group.shapes)
    grads = synth.grads_host(group, seed)
    ref = oracle.rs_reduce(world, group.shapes, grads, 1).view(np.uint32).reshape(world, L.Ns)
    tree = oracle.rs_reduce_tree(world, group.shapes, grads, 0).view(np.uint32).reshape(world, L.Ns)
    ag_ref = oracle.ag_copyout(world, group.shapes, synth.ag_host(group, L.Ns, seed).reshape(-1))
    for r in range(world):
        assert np.array_equal(np.load(tmp_path / f"rs_{r}.npy").view(np.uint32), ref[r])
        assert np.array_equal(np.load(tmp_path / f"tree_{r}.npy").view(np.uint32), tree[r])
        for name in ("sm", "ce"):
            for i in range(group.n_params):
                assert np.array_equal(np.load(tmp_path / f"ag_{name}_{r}_{i}.npy"), ag_ref[i])
