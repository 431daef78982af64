"""Process bodies for the exchange tests: n processes share one GPU, each holding W/n ranks'
gradients and all-gather shards in its two arenas, and reach the others' arenas through the
library's CUDA IPC calls (fsdp2_layout_aware_b200.exchange).  They meet only at gloo barriers."""
import datetime
import os

import numpy as np


def exchange_worker(proc, n_procs, port, shapes, world, seed, out_dir):
    import torch
    import torch.distributed as dist

    import synth
    from fsdp2_layout_aware_b200 import exchange as X
    from fsdp2_layout_aware_b200 import tide as T
    from synth import configs
    from _gpu_helpers import bits_of, to_dev

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=proc, world_size=n_procs,
                            timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        group = configs.Group("exchange", world, tuple(shapes))
        full = T.Plan(group.shapes, world)
        Ns = full.shard_numel
        lay = X.arena_layout(group.shapes, world, n_procs, Ns)
        mine = list(X.ranks_of(proc, world, n_procs))
        grads = torch.full((lay.grad_elems,), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        shards = torch.full((lay.shard_elems,), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        ag = synth.ag_host(group, Ns, seed).reshape(world, Ns)
        for j, k in enumerate(mine):
            for i in range(group.n_params):
                o = j * lay.grad_stride + lay.grad_off[i]
                if lay.numel[i]:
                    grads[o: o + lay.numel[i]] = to_dev(synth.grad_host(group, seed, k, i))
            row = ag[k].copy()
            for i in range(group.n_params):      # pads of the shard are poisoned: never read
                c = full.query(i)["chunk_numel"]
                valid = max(0, min(c, group.numel(i) - k * c))
                off = full.query(i)["shard_offset"]
                row[off + valid: off + c] = 0xFFFF
            if Ns:
                shards[j * lay.shard_stride: j * lay.shard_stride + Ns] = to_dev(row)
        torch.cuda.synchronize()
        dist.barrier()                                       # every arena is filled
        exports = X.all_exports(X.export({"grads": grads, "shards": shards}))
        peers = X.PeerMaps(exports, proc, 0, {"grads": grads.data_ptr(), "shards": shards.data_ptr()})
        try:
            gp, gn = X.grad_table(lay, world, n_procs, peers.bases("grads", n_procs))
            gtab = T.PointerTable(gp, gn, keep=[grads])
            stab = T.PointerTable(X.shard_table(lay, world, n_procs, peers.bases("shards", n_procs)),
                                  [Ns] * world, keep=[shards])
            outs, trees, pipes = {}, {}, {}
            for k in mine:
                plan = T.Plan(group.shapes, world, rank=k)
                outs[k] = torch.full((Ns,), float("nan"), device="cuda")
                plan.rs_reduce(gtab, outs[k], scale_mode=T.TIDE_SCALE_INV_WORLD)
                trees[k] = torch.full((Ns,), float("nan"), device="cuda")
                plan.rs_reduce(gtab, trees[k], scale_mode=T.TIDE_SCALE_NONE, order=T.TIDE_ORDER_TREE)
                # the same shard with the copy engines pulling row k of every rank's gradients
                # (peers' included) into local slots, reduced segment by segment on the SMs
                rows = [torch.full((Ns,), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
                        for _ in range(world)]
                pipes[k] = torch.full((Ns,), float("nan"), device="cuda")
                plan.rs_reduce_pipelined(gtab, pipes[k], rows, min(3, world), torch.cuda.Stream(),
                                         scale_mode=T.TIDE_SCALE_INV_WORLD)
                torch.cuda.synchronize()
                plan.check()
            placed = {}
            for engine, name in ((T.TIDE_ENGINE_SM, "sm"), (T.TIDE_ENGINE_CE, "ce")):
                params = [torch.full((full.query(i)["padded_numel"],), 0x7777, dtype=torch.int16,
                                     device="cuda").view(torch.bfloat16) for i in range(group.n_params)]
                full.ag_gather_place(stab, params, engine=engine)
                placed[name] = params
            torch.cuda.synchronize()
            full.check()
            for k in mine:
                np.save(os.path.join(out_dir, f"rs_{k}.npy"), outs[k].cpu().numpy())
                np.save(os.path.join(out_dir, f"tree_{k}.npy"), trees[k].cpu().numpy())
                np.save(os.path.join(out_dir, f"pipe_{k}.npy"), pipes[k].cpu().numpy())
            for name, params in placed.items():
                for i, p in enumerate(params):
                    np.save(os.path.join(out_dir, f"ag_{name}_{proc}_{i}.npy"), bits_of(p))
        finally:
            torch.cuda.synchronize()
            dist.barrier()                                   # no process still reads a peer
            peers.close()
            dist.barrier()                                   # every mapping gone before frees
    finally:
        dist.destroy_process_group()


def ipc_worker(proc, port, out_dir):
    """Process 0 exports a buffer at an offset inside its allocation; process 1 maps it with
    tide_ipc_open, reads it with a copy, and writes a pattern back through the mapping."""
    import torch
    import torch.distributed as dist
    from fsdp2_layout_aware_b200 import tide as T

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=proc, world_size=2, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        if proc == 0:
            big = torch.arange(1 << 20, dtype=torch.int32, device="cuda")
            view = big[1000:]
            st, handle, off, dev = T.tide_ipc_export(view.data_ptr())
            assert st == T.TIDE_OK and dev == 0 and off % 4 == 0
            torch.cuda.synchronize()
            obj = [(handle, off)]
            dist.broadcast_object_list(obj, src=0)
            dist.barrier()                               # process 1 has read and written
            torch.cuda.synchronize()
            np.save(os.path.join(out_dir, "owner_after.npy"), big[:2048].cpu().numpy())
            dist.barrier()
        else:
            obj = [None]
            dist.broadcast_object_list(obj, src=0)
            handle, off = obj[0]
            st, base = T.tide_ipc_open(handle, 0)
            assert st == T.TIDE_OK and base != 0
            # a zero-copy tensor over the mapped view (same GPU: the mapping is not a peer's)
            class _View:
                def __init__(self, ptr, n):
                    self.__cuda_array_interface__ = {"data": (ptr, False), "shape": (n,),
                                                     "typestr": "<i4", "version": 3}
            mapped = torch.as_tensor(_View(base + off, 32), device="cuda")
            np.save(os.path.join(out_dir, "peer_read.npy"), mapped[:16].clone().cpu().numpy())
            mapped[16:24].fill_(-5)
            torch.cuda.synchronize()
            dist.barrier()
            dist.barrier()
            del mapped
            assert T.tide_ipc_close(base, 0) == T.TIDE_OK
    finally:
        dist.destroy_process_group()
