"""The layout readings pinned against FSDP2 itself (CPU, gloo).

A real FSDP2 job (fully_shard, bf16 parameters, fp32 reduction) runs over W processes.
Its collectives are wrapped to capture the buffers FSDP2 builds. The checks:
- FSDP2's all-gather buffer, put through the oracle's copy-out, gives back the full
  parameters. Its length is the plan's W*Ns.
- FSDP2's packed fp32 gradient buffer of each rank equals the oracle's pack.
- Its reduce-scatter output equals the oracle's reduce-scatter. The inputs are exactly
  summable, so the collective's order of adds does not matter.
"""
import os

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
from fsdp2_layout_aware_b200 import tide as T

from _dist_helpers import free_port
from _fsdp2_workers import fsdp2_worker, integer_grads, param_values

pytest.importorskip("torch.distributed.fsdp._fully_shard._fsdp_collectives")

SHAPES = ((37, 16), (1000,), (7, 3), (5, 130), (64, 8))


def bf16_bits(a):
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


@pytest.mark.parametrize("world", [2, 3])
def test_fsdp2_buffers_match_the_layout_and_the_oracle(world, tmp_path):
    mp.spawn(fsdp2_worker, args=(world, free_port(), SHAPES, str(tmp_path)), nprocs=world, join=True)
    L = oracle.layout(world, SHAPES)
    plan = T.Plan(SHAPES, world, host_only=True)
    assert plan.shard_numel == L.Ns
    full = param_values(SHAPES)
    grads = [[bf16_bits(g).reshape(-1) for g in integer_grads(SHAPES, k)] for k in range(world)]
    rs = oracle.rs_reduce(world, SHAPES, grads, 0).reshape(world, L.Ns)
    for r in range(world):
        ag = np.load(tmp_path / f"ag_{r}.npy")
        assert ag.size == world * L.Ns                       # FSDP2's buffer is [W][Ns]
        placed = oracle.ag_copyout(world, SHAPES, ag)
        for i, p in enumerate(full):
            n = p.size
            assert np.array_equal(placed[i][:n], bf16_bits(p).reshape(-1)), (r, i)
        packed = np.load(tmp_path / f"rs_in_{r}.npy")
        assert np.array_equal(packed.view(np.uint32),
                              oracle.pack_f32(world, SHAPES, grads[r]).view(np.uint32)), r
        out = np.load(tmp_path / f"rs_out_{r}.npy")
        assert np.array_equal(out.view(np.uint32), rs[r].view(np.uint32)), r
    # TIDE's tiles cover exactly those shards
    for t in plan.tiles():
        assert 0 <= t.dst_off - t.rank * L.Ns < L.Ns


def test_fsdp2_bf16_pack_is_the_slot_reuse_staging(tmp_path):
    """With a bf16 reduction FSDP2 packs each rank's gradients, still bf16, into the
    rank-major layout: that is Slot-Reuse staging (the oracle's slot_stage), pads as +0."""
    world = 3
    mp.spawn(fsdp2_worker, args=(world, free_port(), SHAPES, str(tmp_path), False), nprocs=world,
             join=True)
    L = oracle.layout(world, SHAPES)
    for r in range(world):
        grads = [bf16_bits(g).reshape(-1) for g in integer_grads(SHAPES, r)]
        slot = np.zeros(world * L.Ns, dtype=np.uint16)           # FSDP2 pads with +0
        oracle.slot_stage(world, SHAPES, grads, slot)
        assert np.array_equal(np.load(tmp_path / f"rs_in_bf16_{r}.npy"), slot), r


def _averaged(world, tmp_path):
    mp.spawn(fsdp2_worker, args=(world, free_port(), SHAPES, str(tmp_path), True, True),
             nprocs=world, join=True)
    L = oracle.layout(world, SHAPES)
    grads = [[bf16_bits(g).reshape(-1) for g in integer_grads(SHAPES, k)] for k in range(world)]
    got, total = [], oracle.rs_reduce(world, SHAPES, grads, 0)
    for r in range(world):
        for i in range(len(SHAPES)):
            c, n = L.c[i], int(np.prod(SHAPES[i]))
            valid = max(0, min(c, n - r * c))
            local = np.load(tmp_path / f"grad_{r}_{i}.npy").reshape(-1)
            assert local.size >= valid
            start = r * L.Ns + L.off[i]
            got.append((local[:valid], start, valid))
    return got, total


@pytest.mark.parametrize("world", [2, 4])
def test_fsdp2_average_is_the_scaled_reduction(world, tmp_path):
    """FSDP2's averaged gradient shard (sum, then its division by W) equals the oracle's
    sum times fl32(1/W) bit for bit: for power-of-two W the two are the same operation."""
    got, _ = _averaged(world, tmp_path)
    grads = [[bf16_bits(g).reshape(-1) for g in integer_grads(SHAPES, k)] for k in range(world)]
    ref = oracle.rs_reduce(world, SHAPES, grads, 1)
    for local, start, valid in got:
        assert np.array_equal(local.view(np.uint32), ref[start: start + valid].view(np.uint32))


def test_fsdp2_average_divides_for_other_world_sizes(tmp_path):
    """For W = 3 FSDP2 divides the sum by 3 (correctly rounded); the oracle's reading
    multiplies by fl32(1/3), which may differ in the last bit."""
    got, total = _averaged(3, tmp_path)
    for local, start, valid in got:
        want = (total[start: start + valid].astype(np.float32) / np.float32(3)).astype(np.float32)
        assert np.array_equal(local.view(np.uint32), want.view(np.uint32))
