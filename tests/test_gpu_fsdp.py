"""Sharded data-parallel training with TIDE's collectives (fsdp2_layout_aware_b200.fsdp).

2 and 3 processes share this GPU, each a rank of a small bf16 network (W=3 pads the 10-row
layers to 12 rows; its (1, 10) output scale leaves every rank but rank 0 only pad rows).  Every step: TIDE-AG places every rank's shard into each rank's
parameters, the module runs forward and backward with autograd writing into the gradient
arena, TIDE-RS reduces each rank's gradient shard from every rank's gradients, and SGD
updates the rank's fp32 master shard.  Checked at every step, bit for bit against the
oracle: the placed parameters (the oracle's copy-out of the rank-major concatenation of all
ranks' shards) and each reduced gradient shard (the oracle's reduce-scatter of all ranks'
saved gradients, x 1/W).  The optimizer step is checked against its own arithmetic.
"""
import numpy as np
import pytest
import torch

import oracle

from _dist_helpers import run_procs

pytestmark = pytest.mark.gpu

SHAPES = ((1, 10), (24, 40), (24,), (10, 24), (10,))    # the module's own parameter first


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_training_steps_match_the_oracle(world, tmp_path):
    from _fsdp_tide_workers import train_worker
    steps, lr = 3, 0.05
    run_procs(train_worker, world, lambda port: (world, port, steps, lr, str(tmp_path), SHAPES))
    L = oracle.layout(world, SHAPES)
    P = len(SHAPES)
    for step in range(steps):
        shards = [np.load(tmp_path / f"shard_{step - 1}_{r}.npy") for r in range(world)] if step else None
        for r in range(world):
            placed = [np.load(tmp_path / f"placed_{step}_{r}_{i}.npy") for i in range(P)]
            if shards is not None:
                want = oracle.ag_copyout(world, SHAPES, np.concatenate(shards))
                for i in range(P):
                    assert np.array_equal(placed[i], want[i]), (step, r, i)
            if r:
                first = [np.load(tmp_path / f"placed_{step}_0_{i}.npy") for i in range(P)]
                assert all(np.array_equal(a, b) for a, b in zip(placed, first))
        grads = [[np.load(tmp_path / f"grad_{step}_{k}_{i}.npy") for i in range(P)] for k in range(world)]
        ref = oracle.rs_reduce(world, SHAPES, grads, 1).reshape(world, L.Ns)
        for r in range(world):
            gs = np.load(tmp_path / f"gshard_{step}_{r}.npy")
            assert np.array_equal(gs.view(np.uint32), ref[r].view(np.uint32)), (step, r)
            m0 = np.load(tmp_path / f"master0_{step}_{r}.npy")
            m1 = np.load(tmp_path / f"master1_{step}_{r}.npy")
            np.testing.assert_allclose(m1, m0 - np.float32(lr) * gs, rtol=1e-6, atol=1e-7)
            sh = np.load(tmp_path / f"shard_{step}_{r}.npy")
            bf = torch.from_numpy(m1).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(sh, bf)
    # the parameters moved: the last shards differ from the first placement's
    first = np.concatenate([np.load(tmp_path / f"placed_0_0_{i}.npy") for i in range(P)])
    last = oracle.ag_copyout(world, SHAPES, np.concatenate(
        [np.load(tmp_path / f"shard_{steps - 1}_{r}.npy") for r in range(world)]))
    assert not np.array_equal(first, np.concatenate(last))
