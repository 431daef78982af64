"""The exchange with one process per rank group, through the library's CUDA IPC calls.

n processes share this one GPU, each holding W/n ranks' gradients and all-gather shards in
two arenas; the others' arenas are mapped with tide_ipc_open and enter the pointer tables.
Each process reduces the shards of the ranks it holds (one-rank plans, rank and tree order)
and places every rank's shard (SM and copy engines), bit for bit against the oracle.  On a
machine with several GPUs the same calls map other GPUs' memory over NVLink; here the mapping
is within one GPU.  No kernel waits on another process: the processes meet only at gloo
barriers.  Also: bench.py's exchange mode under torchrun, two processes on this GPU.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import configs

from _dist_helpers import free_port, run_procs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = ((37, 16), (1000,), (7, 3), (5, 130), (64, 64), (8 * 4 + 3, 40), (0, 5), (256, 256))


def test_ipc_export_open_read_write(tmp_path):
    from _exchange_workers import ipc_worker
    run_procs(ipc_worker, 2, lambda port: (port, str(tmp_path)))
    assert np.array_equal(np.load(tmp_path / "peer_read.npy"), np.arange(1000, 1016, dtype=np.int32))
    after = np.load(tmp_path / "owner_after.npy")
    want = np.arange(2048, dtype=np.int32)
    want[1016:1024] = -5
    assert np.array_equal(after, want)


@pytest.mark.parametrize("world,n_procs", [(2, 2), (4, 2), (8, 4), (3, 3)])
def test_exchange_over_ipc_matches_oracle(world, n_procs, tmp_path):
    from _exchange_workers import exchange_worker
    seed = 74
    run_procs(exchange_worker, n_procs,
         lambda port: (n_procs, port, SHAPES, world, seed, str(tmp_path)))
    group = configs.Group("exchange", world, SHAPES)
    L = oracle.layout(world, group.shapes)
    grads = synth.grads_host(group, seed)
    ref = oracle.rs_reduce(world, group.shapes, grads, 1).view(np.uint32).reshape(world, L.Ns)
    tree = oracle.rs_reduce_tree(world, group.shapes, grads, 0).view(np.uint32).reshape(world, L.Ns)
    ag_ref = oracle.ag_copyout(world, group.shapes, synth.ag_host(group, L.Ns, seed).reshape(-1))
    for k in range(world):
        assert np.array_equal(np.load(tmp_path / f"rs_{k}.npy").view(np.uint32), ref[k]), k
        assert np.array_equal(np.load(tmp_path / f"tree_{k}.npy").view(np.uint32), tree[k]), k
        assert np.array_equal(np.load(tmp_path / f"pipe_{k}.npy").view(np.uint32), ref[k]), k
    for p in range(n_procs):
        for name in ("sm", "ce"):
            for i in range(group.n_params):
                assert np.array_equal(np.load(tmp_path / f"ag_{name}_{p}_{i}.npy"), ag_ref[i]), (p, name, i)


def test_bench_exchange_mode_two_processes_on_one_gpu():
    """bench.py --gpus 2 under torchrun: the exchange mode runs and prints one line."""
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--steps", "3", "--warmup", "1", "--workload", "tiny", "--e2e-steps", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["value"] > 0 and d["scaling"] == "strong"
    assert "exchange" in d["config"]["parallelism"] and d["e2e"]["value"] > 0
    assert d["roofline"]["bound"] == "hbm" and d["gpu_launches"] == 3 * (1 + 2)   # shared GPU


def test_bench_exchange_mode_one_process_with_nccl():
    """bench.py --mode exchange in one process: a one-process NCCL group holding every rank;
    the step, the end-to-end run and the NCCL reduce-scatter comparison all complete."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--mode", "exchange", "--steps", "3",
           "--warmup", "1", "--workload", "tiny", "--e2e-steps", "1"]
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["n_gpus"] == 1 and d["value"] > 0 and d["e2e"]["value"] > 0
    nc = d["nccl_compare"]
    assert "error" not in nc, nc
    assert nc["stock_ms"]["nccl_reduce_scatter"] > 0 and nc["tide_rs_ms"] > 0
    assert set(nc["gemm_slowdown"]) == {"nccl_reduce_scatter", "tide_rs",
                                        "tide_rs_short_ctas_gemm_high_priority", "tide_rs_4_ctas"}
