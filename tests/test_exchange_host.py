"""The exchange across processes, host side (no GPU): rank placement, arena layout, pointer
tables, and the handle exchange over a gloo process group with fake mappings.

Each process holds W/n consecutive ranks; every process must end up with the same table
entries, each pointing at the owner's arena (its own address locally, the mapped address of
the owner's export elsewhere), and must open each peer allocation exactly once.
"""
import json
import os

import pytest
import torch.multiprocessing as mp

import oracle
from fsdp2_layout_aware_b200 import exchange as X
from fsdp2_layout_aware_b200 import tide as T
from synth import configs

from _dist_helpers import free_port


@pytest.mark.parametrize("world,n", [(8, 1), (8, 2), (8, 4), (8, 8), (16, 8), (64, 4), (3, 3)])
def test_ranks_are_spread_evenly_and_owned_once(world, n):
    seen = []
    for p in range(n):
        r = X.ranks_of(p, world, n)
        assert len(r) == world // n
        assert all(X.owner_of(k, world, n) == p for k in r)
        seen += list(r)
    assert seen == list(range(world))


def test_uneven_spread_is_refused():
    with pytest.raises(ValueError):
        X.ranks_of(0, 8, 3)
    with pytest.raises(ValueError):
        X.ranks_of(4, 8, 4)


def test_arena_layout_aligns_every_param_and_shard():
    g = configs.tiny()
    L = oracle.layout(g.world, g.shapes)
    lay = X.arena_layout(g.shapes, g.world, 2, L.Ns)
    assert lay.per_proc == 2
    assert list(lay.numel) == [g.numel(i) for i in range(g.n_params)]
    for i in range(g.n_params):
        assert lay.grad_off[i] % X.ALIGN_ELEMS == 0
        if i + 1 < g.n_params:
            assert lay.grad_off[i + 1] >= lay.grad_off[i] + lay.numel[i]
    assert lay.grad_stride % X.ALIGN_ELEMS == 0 and lay.grad_stride >= lay.grad_off[-1] + lay.numel[-1]
    assert lay.shard_stride % X.ALIGN_ELEMS == 0 and lay.shard_stride >= L.Ns
    assert lay.grad_elems == 2 * lay.grad_stride and lay.shard_elems == 2 * lay.shard_stride


def test_tables_point_into_the_owners_arenas():
    g = configs.qwen3moe(4)
    W, P, n = g.world, g.n_params, 4
    lay = X.arena_layout(g.shapes, W, n, 1000)
    gbase = [10 ** 12 * (p + 1) for p in range(n)]
    sbase = [10 ** 13 * (p + 1) for p in range(n)]
    ptrs, numels = X.grad_table(lay, W, n, gbase)
    assert len(ptrs) == W * P
    for k in range(W):
        p, j = k // (W // n), k % (W // n)
        for i in range(P):
            assert ptrs[k * P + i] == gbase[p] + 2 * (j * lay.grad_stride + lay.grad_off[i])
            assert numels[k * P + i] == g.numel(i)
    sh = X.shard_table(lay, W, n, sbase)
    assert sh == [sbase[r // 2] + 2 * (r % 2) * lay.shard_stride for r in range(W)]
    # no two gradient views of one arena overlap
    spans = sorted((a, a + 2 * m) for a, m in zip(ptrs, numels))
    assert all(spans[t][1] <= spans[t + 1][0] for t in range(len(spans) - 1))


def _fake_base(handle: bytes) -> int:
    return int.from_bytes(handle[:8], "little") * 2 ** 24


def _exchange_worker(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = configs.Group("x", 8, ((37, 16), (1000,), (7, 3), (64, 64)))
        lay = X.arena_layout(g.shapes, g.world, world, 5000)
        # this process's arenas: fake local addresses, and fake handles naming the process;
        # both arenas sit in one allocation, as they may in a caching allocator
        local = {"grads": 7 * 2 ** 40 + rank * 2 ** 32, "shards": 7 * 2 ** 40 + rank * 2 ** 32 + 2 ** 30}
        handle = bytes([rank + 1]) + bytes(T.TIDE_IPC_HANDLE_BYTES - 1)
        mine = {"grads": (handle, 4096), "shards": (handle, 4096 + 2 ** 20)}
        exports = X.all_exports(mine)
        opened, closed = [], []

        def opener(h, device):
            opened.append(h)
            return T.TIDE_OK, _fake_base(h)

        def closer(base, device):
            closed.append(base)
            return T.TIDE_OK

        peers = X.PeerMaps(exports, rank, 0, local, opener=opener, closer=closer)
        ptrs, _ = X.grad_table(lay, g.world, world, peers.bases("grads", world))
        shards = X.shard_table(lay, g.world, world, peers.bases("shards", world))
        peers.close()
        with open(os.path.join(out_dir, f"x_{rank}.json"), "w") as f:
            json.dump({"ptrs": ptrs, "shards": shards, "opened": len(opened),
                       "distinct": len(set(opened)), "closed": len(closed)}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_handle_exchange_over_gloo(world, tmp_path):
    mp.spawn(_exchange_worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"x_{r}.json")) for r in range(world)]
    g = configs.Group("x", 8, ((37, 16), (1000,), (7, 3), (64, 64)))
    lay = X.arena_layout(g.shapes, g.world, world, 5000)
    P = g.n_params
    for me, d in enumerate(res):
        assert d["opened"] == d["distinct"] == world - 1 == d["closed"]   # one map per peer
        for k in range(g.world):
            p = X.owner_of(k, g.world, world)
            j = k - p * lay.per_proc
            if p == me:
                gb = 7 * 2 ** 40 + me * 2 ** 32
                sb = gb + 2 ** 30
            else:
                base = _fake_base(bytes([p + 1]) + bytes(T.TIDE_IPC_HANDLE_BYTES - 1))
                gb, sb = base + 4096, base + 4096 + 2 ** 20
            for i in range(P):
                assert d["ptrs"][k * P + i] == gb + 2 * (j * lay.grad_stride + lay.grad_off[i])
            assert d["shards"][k] == sb + 2 * j * lay.shard_stride


def test_exchange_bytes_add_up_to_the_single_gpu_step():
    """Over all processes, RS bytes equal the single-GPU RS; each GPU places every shard."""
    import bench
    g = configs.llama70b()
    L = oracle.layout(g.world, g.shapes)
    B1 = bench.alg_bytes(g, L)
    for n in (2, 4, 8):
        parts = [bench.exchange_bytes(g, L.c, L.Ns, X.ranks_of(p, g.world, n), n) for p in range(n)]
        assert sum(b["rs"] for b in parts) == B1["rs"]
        assert all(b["ag"] == B1["ag"] for b in parts)
        per = g.world // n
        # NVLink: the share of each read held by other processes
        assert sum(b["rs_nvlink"] for b in parts) == B1["rs_read"] * (g.world - per) // g.world
        assert all(b["ag_nvlink"] == B1["ag_read"] * (g.world - per) // g.world for b in parts)


def test_a_peer_allocation_is_mapped_once_and_unmapped_after_its_last_user(monkeypatch):
    """CUDA maps an IPC handle at most once per process and device, and several arenas (of
    different parameter groups) may share one allocation: open_shared hands later users the
    first mapping and close_shared unmaps only after the last of them."""
    calls = []

    def fake_open(handle, device):
        calls.append(("open", bytes(handle), device))
        return T.TIDE_OK, 0x1000 * (len(calls) + 1)

    def fake_close(base, device):
        calls.append(("close", base, device))
        return T.TIDE_OK

    monkeypatch.setattr(T, "tide_ipc_open", fake_open)
    monkeypatch.setattr(T, "tide_ipc_close", fake_close)
    monkeypatch.setattr(X, "_MAPPED", {})
    h1, h2 = b"a" * T.TIDE_IPC_HANDLE_BYTES, b"b" * T.TIDE_IPC_HANDLE_BYTES
    st, b1 = X.open_shared(h1, 0)
    st2, b1_again = X.open_shared(h1, 0)
    st3, b2 = X.open_shared(h2, 0)
    st4, b1_other_device = X.open_shared(h1, 1)
    assert st == st2 == st3 == st4 == T.TIDE_OK
    assert b1 == b1_again and len({b1, b2, b1_other_device}) == 3
    assert [c[0] for c in calls] == ["open", "open", "open"]
    assert X.close_shared(b1, 0) == T.TIDE_OK            # one user of h1 on device 0 remains
    assert [c[0] for c in calls].count("close") == 0
    assert X.close_shared(b1, 0) == T.TIDE_OK            # the last one: unmapped now
    assert calls[-1] == ("close", b1, 0)
    X.close_shared(b2, 0)
    X.close_shared(b1_other_device, 1)
    assert X._MAPPED == {}
    # two PeerMaps over exports that share an allocation open it once between them
    exports = [{"arena": (h1, 0)}, {"arena": (h1, 4096)}]
    calls.clear()
    m1 = X.PeerMaps(exports[:1] + [{"arena": (h2, 0)}], 1, 0, {"arena": 0xAAAA})
    m2 = X.PeerMaps([{"arena": (h1, 256)}, {"arena": (h2, 0)}], 1, 0, {"arena": 0xBBBB})
    assert [c[0] for c in calls] == ["open"]
    assert m2.bases("arena", 2)[0] == m1.bases("arena", 2)[0] + 256
    m1.close()
    assert [c[0] for c in calls] == ["open"]
    m2.close()
    assert [c[0] for c in calls] == ["open", "close"]
