"""FSDP2's own fully_shard with TIDE's all-gather and reduce-scatter (fsdp2_layout_aware_b200.fsdp2).

2 and 3 processes share this GPU, each a rank of FSDP2 (bf16 compute parameters, fp32
reduction, fp32 master parameters, SGD) over a small network, sharded per layer and at the
root.  FSDP2's copy-out runs as tide_ag_gather_place from every rank's arena, its fp32 pack
as tide_rs_stage_one into the rank's own arena, its reduce-scatter as tide_rs_reduce_slots.
Checked bit for bit against the oracle at every call of every step:
  * each placement: the padded parameters each rank placed equal the oracle's copy-out of
    the rank-major concatenation of the rows all ranks had copied in;
  * each staging: the rank's arena equals the oracle's staging of the rank's gradients (at
    valid positions; pads keep what they held);
  * each reduction: the rank's fp32 shard equals rows r of the oracle's reduce-scatter of all
    ranks' gradients, x fl32(1/W) (FSDP2 asks for an average).
"""
import json

import numpy as np
import pytest

import oracle

from _dist_helpers import run_procs

pytestmark = pytest.mark.gpu

pytest.importorskip("torch.distributed.fsdp._fully_shard._fsdp_collectives")


def _load(tmp, name):
    return np.load(tmp / name)


@pytest.mark.parametrize("world,engine,order,mode",
                         [(2, 0, 0, "plain"), (3, 0, 0, "plain"), (3, 1, 1, "plain"),
                          (2, 0, 0, "frozen"), (2, 1, 0, "accum"), (3, 0, 1, "no_reshard"),
                          (3, 0, 0, "accum_unsynced"), (2, 1, 1, "accum_unsynced")],
                         ids=["w2_sm_rank", "w3_sm_rank", "w3_ce_tree", "w2_frozen_param",
                              "w2_ce_rank_grad_accumulation", "w3_sm_tree_no_reshard",
                              "w3_sm_rank_accumulation_sync_off", "w2_ce_tree_accumulation_sync_off"])
def test_fully_shard_with_tide_collectives_matches_the_oracle(world, engine, order, mode, tmp_path):
    """(With a frozen parameter its group stages and reduces the others only, in the layout
    their shapes give; accumulating, each of a step's two micro-batches is reduced; kept
    unsharded after forward, each group is placed once a step; accumulating with gradient
    sync off, FSDP2 packs fp32 gradients, staged into fp32 slots and reduced in rank order.)"""
    from _fsdp2_tide_workers import fsdp2_tide_worker
    steps, lr = 3, 0.05
    run_procs(fsdp2_tide_worker, world,
              lambda port: (world, port, steps, lr, str(tmp_path), engine, order, mode))
    per_step = 2 if mode == "accum" else 1
    shapes = [[tuple(s) for s in g] for g in json.loads((tmp_path / "shapes.json").read_text())]
    counts = [json.loads((tmp_path / f"counts_{r}.json").read_text()) for r in range(world)]
    assert all({k: v for k, v in c.items() if k != "losses"} ==
               {k: v for k, v in counts[0].items() if k != "losses"} for c in counts)
    rs_oracle = oracle.rs_reduce if order == 0 else oracle.rs_reduce_tree
    for g, S in enumerate(shapes):
        L = oracle.layout(world, S)
        P = len(S)
        n_place = counts[0][f"place_{g}"]
        n_reduce = counts[0][f"reduce_{g}"]
        assert n_place >= steps * per_step and n_reduce == steps * per_step
        assert counts[0][f"stage_{g}"] == n_reduce
        for n in range(n_place):
            ag = np.concatenate([_load(tmp_path, f"row_{g}_{n}_{k}.npy") for k in range(world)])
            want = oracle.ag_copyout(world, S, ag)
            for r in range(world):
                for i in range(P):
                    got = _load(tmp_path, f"placed_{g}_{n}_{r}_{i}.npy")
                    assert np.array_equal(got, want[i]), (g, n, r, i)
        for n in range(n_reduce):
            staged = json.loads((tmp_path / f"staged_shapes_{g}_{n}.json").read_text())
            Sr, f32 = [tuple(x) for x in staged["shapes"]], staged["f32"]
            assert f32 == (mode == "accum_unsynced")
            Lr = oracle.layout(world, Sr)
            grads = [[_load(tmp_path, f"grad_{g}_{n}_{k}_{i}.npy") for i in range(len(Sr))]
                     for k in range(world)]
            for k in range(world):
                exp = _load(tmp_path, f"slot0_{g}_{n}_{k}.npy").copy()
                (oracle.slot_stage_f32 if f32 else oracle.slot_stage)(world, Sr, grads[k],
                                                                      exp[:world * Lr.Ns])
                assert np.array_equal(_load(tmp_path, f"slot1_{g}_{n}_{k}.npy"), exp), (g, n, k)
            ref = (oracle.rs_reduce_f32 if f32 else rs_oracle)(world, Sr, grads, 1).reshape(world, Lr.Ns)
            for r in range(world):
                got = _load(tmp_path, f"shard_{g}_{n}_{r}.npy")
                assert np.array_equal(got.view(np.uint32), ref[r].view(np.uint32)), (g, n, r)
    # training moved the parameters: the last placement of each group differs from the first
    for g, S in enumerate(shapes):
        last = counts[0][f"place_{g}"] - 1
        first = np.concatenate([_load(tmp_path, f"placed_{g}_0_0_{i}.npy") for i in range(len(S))])
        final = np.concatenate([_load(tmp_path, f"placed_{g}_{last}_0_{i}.npy") for i in range(len(S))])
        assert not np.array_equal(first, final), g
