"""Process body for the cross-process flag test: two processes share one GPU.  Every wait finds
its flag already set by the other process (which finished and met this one at a host barrier
first) or runs out its time limit on a flag nothing sets; no kernel waits on one that runs at
the same time."""
import datetime
import json
import os


def flag_worker(proc, port, out_dir):
    import torch
    import torch.distributed as dist
    from fsdp2_layout_aware_b200 import exchange as X
    from fsdp2_layout_aware_b200 import tide as T

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=proc, world_size=2, timeout=datetime.timedelta(seconds=120))
    res = {}
    try:
        torch.cuda.set_device(0)
        flags = torch.zeros(2, dtype=torch.int32, device="cuda")
        status = torch.full((1,), -7, dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        exports = X.all_exports(X.export({"flags": flags}))
        peers = X.PeerMaps(exports, proc, 0, {"flags": flags.data_ptr()})
        p0 = peers.bases("flags", 2)[0]                          # process 0's flags, in this process
        if proc == 0:
            res["signal"] = T.tide_flag_signal(p0, 5)            # its own flag 0
        torch.cuda.synchronize()
        dist.barrier()
        if proc == 1:
            res["wait_set"] = T.tide_flag_wait([p0], 5, 10**9, status.data_ptr())
            torch.cuda.synchronize()
            res["status_set"] = int(status.item())
            res["wait_unset"] = T.tide_flag_wait([p0, p0 + 4], 1, 20 * 10**6, status.data_ptr())
            torch.cuda.synchronize()
            res["status_unset"] = int(status.item())
            res["signal_peer"] = T.tide_flag_signal(p0 + 4, 9)   # process 0's flag 1, through the mapping
        torch.cuda.synchronize()
        dist.barrier()
        if proc == 0:
            res["wait_own"] = T.tide_flag_wait([p0, p0 + 4], 5, 10**9, status.data_ptr())
            torch.cuda.synchronize()
            res["status_own"] = int(status.item())
            res["flags"] = flags.tolist()
        torch.cuda.synchronize()
        dist.barrier()
        peers.close()
        dist.barrier()
        with open(os.path.join(out_dir, f"flags_{proc}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()
