"""FSDP2's side of fsdp2_layout_aware_b200.fsdp2, on the CPU.

FSDP2 (fully_shard, bf16 compute, fp32 reduction, SGD) runs over 2 and 3 gloo processes
twice: stock, and with TIDE's all-gather and reduce-scatter comms plus the copy-out and pack
routed to TIDE groups, whose data movement is the oracle's (placement, Slot-Reuse staging,
slot reduction x fl32(1/W)) with gloo standing in for the peer reads.  The sharded gradients
of every step and the final parameters must be stock FSDP2's: bit for bit at W = 2 (one add,
and 1/2 is exact), within fp32 rounding of a reordered 3-term sum at W = 3.  Every TIDE group
must have seen each placement, staging and reduction FSDP2 should ask for.
"""
import json

import numpy as np
import pytest

from _dist_helpers import run_procs

pytest.importorskip("torch.distributed.fsdp._fully_shard._fsdp_collectives")


# The calls each TIDE group sees per step, in fully_shard order: l1, l2, then the root.
# Resharded after forward, l1 and l2 are placed again in backward; the root stays unsharded
# from forward to backward.  Accumulating over two micro-batches, each is reduce-scattered.
# Kept unsharded after forward, every group is placed once.
CALLS = {
    "plain": (["place", "place", "stage", "reduce"], ["place", "stage", "reduce"]),
    "frozen": (["place", "place", "stage", "reduce"], ["place", "stage", "reduce"]),
    "accum": (["place", "place", "stage", "reduce"] * 2, ["place", "stage", "reduce"] * 2),
    "no_reshard": (["place", "stage", "reduce"], ["place", "stage", "reduce"]),
    "accum_unsynced": (["place", "place", "place", "place", "stage", "reduce"],
                       ["place", "place", "stage", "reduce"]),
}


@pytest.mark.parametrize("world,mode", [(2, "plain"), (3, "plain"), (2, "frozen"), (2, "accum"),
                                        (3, "no_reshard"), (2, "accum_unsynced"), (3, "accum_unsynced")],
                         ids=["w2", "w3", "w2_frozen_param", "w2_grad_accumulation",
                              "w3_no_reshard_after_forward", "w2_accumulation_sync_off",
                              "w3_accumulation_sync_off"])
def test_fsdp2_with_tide_comms_gives_stock_fsdp2_results(world, mode, tmp_path):
    """With a frozen parameter (no gradient) its group reduce-scatters the others only; with
    gradient accumulation the reduced gradients are the sum over both micro-batches (sync off:
    FSDP2 packs fp32 gradients, staged into the fp32 slots)."""
    from _fsdp2_tide_workers import fsdp2_oracle_worker
    steps, lr = 3, 0.05
    run_procs(fsdp2_oracle_worker, world,
              lambda port: (world, port, steps, lr, str(tmp_path), mode))
    trained = [0, 1, 3, 4] if mode == "frozen" else list(range(5))  # scale, l1.w, l1.b, ...
    for r in range(world):
        names = [f"grad_{s}_{r}_{i}" for s in range(steps) for i in trained] + \
                [f"param_{r}_{i}" for i in range(5)]
        for name in names:
            a, b = np.load(tmp_path / f"stock_{name}.npy"), np.load(tmp_path / f"tide_{name}.npy")
            assert a.shape == b.shape, name
            if world == 2:
                assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), name
            else:
                np.testing.assert_allclose(b, a, rtol=1e-5, atol=1e-7, err_msg=name)
        calls = json.loads((tmp_path / f"calls_{r}.json").read_text())
        inner, root = CALLS[mode]
        assert calls[0] == calls[1] == inner * steps, calls
        assert calls[2] == root * steps, calls


def test_staging_takes_bf16_or_fp32_gradients_of_one_dtype():
    import torch
    from fsdp2_layout_aware_b200 import fsdp2 as F
    bf, f32 = torch.zeros(4, 3, dtype=torch.bfloat16), torch.zeros(4, 3)
    assert F._check_grads([bf, bf], 2) is False
    assert F._check_grads([f32], 2) is True
    for bad, n in (([bf, f32], 2), ([torch.zeros(3, dtype=torch.float16)], 1), ([bf, bf, bf], 2),
                   ([], 2), ([torch.zeros(4, 6, dtype=torch.bfloat16)[:, :3]], 1),
                   ([torch.zeros((), dtype=torch.bfloat16)], 1)):
        with pytest.raises(ValueError):
            F._check_grads(bad, n)


def test_tide_comms_hand_out_the_groups_buffers_and_refuse_others():
    """The all-gather buffer FSDP2 asks for is the group's arena; the reduce-scatter's fp32
    [W][Ns] input is one element expanded to that shape (never materialized) and its [Ns]
    output a fresh fp32 tensor; any other request is refused."""
    import types

    import torch
    from fsdp2_layout_aware_b200 import fsdp2 as F

    W, Ns = 3, 40
    tg = types.SimpleNamespace(world=W, shard_numel=Ns, device=torch.device("cpu"),
                               arena=torch.zeros(W * Ns, dtype=torch.bfloat16),
                               rs_input=torch.zeros(1), reduced=[], pending=None)
    tg.reduce = lambda out, op: tg.reduced.append((out.numel(), op))
    tg.meet = lambda: None
    ag_cls, rs_cls = F._comm_classes()
    ag, rs = ag_cls(tg), rs_cls(tg)
    buf = ag.allocate((W * Ns,), dtype=torch.bfloat16, device=tg.device)
    assert buf.data_ptr() == tg.arena.data_ptr()
    with pytest.raises(ValueError):
        ag.allocate((W * Ns + 1,), dtype=torch.bfloat16, device=tg.device)
    with pytest.raises(ValueError):
        ag.allocate((W * Ns,), dtype=torch.float32, device=tg.device)
    assert ag(buf, buf[:Ns], group=None) is None
    with pytest.raises(ValueError):
        ag(torch.zeros(W * Ns, dtype=torch.bfloat16), buf[:Ns], group=None)
    # before staging FSDP2 asks for the packed input: any [W][n] up to the group's
    inp = rs.allocate((W * Ns,), dtype=torch.float32, device=tg.device)
    assert inp.shape == (W * Ns,) and inp.stride() == (0,) and inp.data_ptr() == tg.rs_input.data_ptr()
    assert inp.view(W, -1).data_ptr() == tg.rs_input.data_ptr()     # FSDP2's pack target
    assert rs.allocate((W * 8,), dtype=torch.float32, device=tg.device).shape == (W * 8,)
    for bad in (W * Ns + W, W * 8 + 1):
        with pytest.raises(ValueError):
            rs.allocate((bad,), dtype=torch.float32, device=tg.device)
    with pytest.raises(ValueError):
        rs.allocate((W * Ns,), dtype=torch.bfloat16, device=tg.device)
    # after staging (its shard numel known) it asks for the output
    tg.pending = (None, Ns)
    out = rs.allocate((Ns,), dtype=torch.float32, device=tg.device)
    assert out.shape == (Ns,) and out.dtype == torch.float32 and out.data_ptr() != inp.data_ptr()
    with pytest.raises(ValueError):
        rs.allocate((Ns + 1,), dtype=torch.float32, device=tg.device)
    import torch.distributed as dist
    assert rs(out, inp, group=None, op=dist.ReduceOp.AVG) is None
    assert tg.reduced == [(Ns, dist.ReduceOp.AVG)]
    with pytest.raises(ValueError):
        rs(out, torch.zeros(W * Ns), group=None, op=dist.ReduceOp.AVG)


def test_resharding_to_a_smaller_world_is_refused():
    """An int reshard_after_forward would all-gather over part of the group in backward;
    TIDE groups refuse it before touching the module."""
    import torch
    from fsdp2_layout_aware_b200 import fsdp2 as F
    m = torch.nn.Linear(4, 4)
    with pytest.raises(ValueError):
        F.fully_shard_tide(m, reshard_after_forward=2)
    assert not hasattr(m, "_tide_group")
