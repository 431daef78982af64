"""fp32 gradients through Slot-Reuse (tide_rs_stage_one_f32, tide_rs_reduce_slots_f32) and read
in place (tide_rs_reduce_f32) against the oracle, bit for bit.

Every source rank stages its fp32 gradients into its own fp32 slot, on the SMs or on the copy
engines (stale contents: NaN, so a pad that is read shows); the slots must equal the oracle's staging word for word (pads keep
the NaN), and the reduction of all ranks' shards (all-rank plan) and of each rank's shard
(one-rank plans) must equal the oracle's fp32 reduction bit for bit, with and without the
1/W scale, on the vector path (32-byte aligned buffers), on the element path (buffers shifted
by one word), and under CTA caps.  The gradients carry bits below bf16 precision.
"""
import numpy as np
import pytest
import torch

import oracle
from fsdp2_layout_aware_b200 import tide as T
from synth import configs

from _gpu_helpers import f32_bits
from _groups import degenerate, mini_sweep, mini_wan, random_group

pytestmark = pytest.mark.gpu

NAN = 0xFFFFFFFF


def groups():
    rng = np.random.default_rng(404)
    return [configs.tiny(), degenerate(), mini_wan(), mini_sweep(2), mini_sweep(8),
            configs.Group("two_tiles", 4, ((4 * 2048 + 3, 9),)),
            random_group(rng, 3, 6, name="rand_w3"), random_group(rng, 5, 5, name="rand_w5"),
            random_group(rng, 64, 4, name="rand_w64"),
            random_group(rng, 256, 3, max_rows=600, name="rand_w256")]


def f32_grads(group, seed):
    """Per rank and param: N(0, 1e-3) in fp32 (not rounded to bf16), every tenth exactly 0."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(group.world):
        row = []
        for i in range(group.n_params):
            g = (rng.standard_normal(group.numel(i)) * 1e-3).astype(np.float32)
            g[::10] = 0.0
            row.append(g)
        out.append(row)
    return out


def dev_f32(arr, shift=0):
    """A device fp32 tensor holding `arr` (float32 or its uint32 words), starting `shift`
    words into a fresh allocation (shift 1: 4-byte but not 32-byte aligned)."""
    words = np.ascontiguousarray(arr).reshape(-1).view(np.int32)
    base = torch.empty(words.size + shift, dtype=torch.int32, device="cuda")
    t = base[shift:]
    t.copy_(torch.from_numpy(words.copy()))
    return t.view(torch.float32)


def stage_all(group, grads, plan, shift, cap=0, engine=T.TIDE_ENGINE_SM):
    W = group.world
    L = oracle.layout(W, group.shapes)
    slots = [dev_f32(np.full(W * L.Ns, NAN, np.uint32), shift) for _ in range(W)]
    for k in range(W):
        g = [dev_f32(grads[k][i], shift) for i in range(group.n_params)]
        plan.rs_stage_one_f32(g, slots[k], engine=engine, max_ctas=cap)
    torch.cuda.synchronize()
    return slots


@pytest.mark.parametrize("engine", [T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE], ids=["sm", "ce"])
@pytest.mark.parametrize("shift", [0, 1], ids=["aligned", "shifted"])
@pytest.mark.parametrize("group", groups(), ids=lambda g: f"{g.name}_w{g.world}")
def test_f32_slot_reuse_matches_the_oracle(group, shift, engine):
    W = group.world
    L = oracle.layout(W, group.shapes)
    grads = f32_grads(group, seed=W * 100 + group.n_params)
    plan = T.Plan(group.shapes, W)
    slots = stage_all(group, grads, plan, shift, engine=engine)
    for k in range(W):
        want = np.full(W * L.Ns, NAN, np.uint32)
        oracle.slot_stage_f32(W, group.shapes, grads[k], want)
        assert np.array_equal(f32_bits(slots[k]), want), k
    host_slots = [f32_bits(s) for s in slots]
    for scale in (0, 1):
        want = oracle.rs_reduce_f32(W, group.shapes, grads, scale).view(np.uint32)
        assert np.array_equal(oracle.rs_reduce_slots_f32(W, group.shapes, host_slots, scale).view(np.uint32),
                              want)
        out = dev_f32(np.full(W * L.Ns, NAN, np.uint32), shift)
        plan.rs_reduce_slots_f32(slots, out, scale_mode=scale)
        torch.cuda.synchronize()
        assert np.array_equal(f32_bits(out), want), scale
        for r in sorted({0, W // 2, W - 1}):
            rp = T.Plan(group.shapes, W, rank=r)
            shard = dev_f32(np.full(L.Ns, NAN, np.uint32), shift)
            rp.rs_reduce_slots_f32(slots, shard, scale_mode=scale)
            torch.cuda.synchronize()
            assert np.array_equal(f32_bits(shard), want[r * L.Ns:(r + 1) * L.Ns]), (scale, r)
            rp.check()
    plan.check()


@pytest.mark.parametrize("shift", [0, 1], ids=["aligned", "shifted"])
@pytest.mark.parametrize("group", groups(), ids=lambda g: f"{g.name}_w{g.world}")
def test_f32_direct_reduce_matches_the_oracle(group, shift):
    """TIDE-RS on fp32 gradients read in place: all shards, and each rank's shard with a
    one-rank plan, bit for bit against the oracle."""
    W = group.world
    L = oracle.layout(W, group.shapes)
    grads = f32_grads(group, seed=W * 31 + group.n_params)
    g = [[dev_f32(grads[k][i], shift) for i in range(group.n_params)] for k in range(W)]
    table = T.TensorTable([t for row in g for t in row])
    plan = T.Plan(group.shapes, W)
    for scale in (0, 1):
        want = oracle.rs_reduce_f32(W, group.shapes, grads, scale).view(np.uint32)
        out = dev_f32(np.full(W * L.Ns, NAN, np.uint32), shift)
        plan.rs_reduce_f32(table, out, scale_mode=scale)
        torch.cuda.synchronize()
        assert np.array_equal(f32_bits(out), want), scale
        assert plan.last_launch()[0] == T.KERNEL_NAMES.index("rs_f32")
        for r in sorted({0, W // 2, W - 1}):
            rp = T.Plan(group.shapes, W, rank=r)
            shard = dev_f32(np.full(L.Ns, NAN, np.uint32), shift)
            rp.rs_reduce_f32(table, shard, scale_mode=scale)
            torch.cuda.synchronize()
            assert np.array_equal(f32_bits(shard), want[r * L.Ns:(r + 1) * L.Ns]), (scale, r)
            rp.check()
    plan.check()


@pytest.mark.parametrize("gshift", range(8))
def test_f32_staging_at_every_relative_alignment(gshift):
    """Gradients shifted by 0..7 words against an aligned slot: the staging copy takes its
    32-byte, 16-byte and word paths (with their heads and tails) and gives the oracle's slot."""
    group = configs.Group("aligns", 4, ((4 * 3000 + 1, 3), (8 * 16 * 4,), (4 * 2048, 4)))
    W = group.world
    L = oracle.layout(W, group.shapes)
    grads = f32_grads(group, seed=60 + gshift)
    plan = T.Plan(group.shapes, W)
    for engine in (T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE):
        slot = dev_f32(np.full(W * L.Ns, NAN, np.uint32), 0)
        g = [dev_f32(grads[1][i], gshift) for i in range(group.n_params)]
        plan.rs_stage_one_f32(g, slot, engine=engine)
        torch.cuda.synchronize()
        want = np.full(W * L.Ns, NAN, np.uint32)
        oracle.slot_stage_f32(W, group.shapes, grads[1], want)
        assert np.array_equal(f32_bits(slot), want), engine
    plan.check()


@pytest.mark.parametrize("cap", [1, 7])
def test_f32_cta_caps_give_the_same_bits(cap):
    group = mini_sweep(8)
    W = group.world
    L = oracle.layout(W, group.shapes)
    grads = f32_grads(group, seed=9)
    plan = T.Plan(group.shapes, W)
    slots = stage_all(group, grads, plan, 0, cap=cap)
    out = torch.empty(W * L.Ns, device="cuda")
    plan.rs_reduce_slots_f32(slots, out, max_ctas=cap)
    torch.cuda.synchronize()
    assert plan.last_launch() == (T.KERNEL_NAMES.index("slot_rs_f32"), cap)
    assert np.array_equal(f32_bits(out), oracle.rs_reduce_f32(W, group.shapes, grads, 1).view(np.uint32))


def test_f32_values_below_bf16_precision_survive():
    """1 + 2^-20 on rank 0, 2^-20 multiples elsewhere: exact sums that bf16 cannot hold."""
    group = configs.Group("fine", 4, ((4 * 8192, 2), (37,)))
    W = group.world
    L = oracle.layout(W, group.shapes)
    rng = np.random.default_rng(3)
    grads = [[((rng.integers(-8, 9, size=group.numel(i)) + (2 ** 20 if k == 0 else 0)) * 2.0 ** -20)
              .astype(np.float32) for i in range(group.n_params)] for k in range(W)]
    plan = T.Plan(group.shapes, W)
    slots = stage_all(group, grads, plan, 0)
    out = torch.empty(W * L.Ns, device="cuda")
    plan.rs_reduce_slots_f32(slots, out, scale_mode=0)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, oracle.rs_reduce_f32(W, group.shapes, grads, 0).astype(np.float64))
    assert np.any(np.abs(got - np.round(got)) > 0)        # the fine bits are there
