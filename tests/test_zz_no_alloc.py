"""tide_rs_reduce_noalloc: the allocation-free reduction, through the C-ABI.

Some callers cannot allocate device memory (for example a runtime whose
caching allocator owns the GPU's memory), so they cannot build a plan, whose
tables tide_plan_group allocates.  tide_rs_reduce_noalloc keeps its tables in
a fixed 1 MiB device array instead.  These tests check that it returns the
same fp32 shards, bit for bit, as tide_rs_reduce on two different groups
called back to back (the shared array is rewritten between them), then on the
first group again with new gradients, and that a group too large for the array
is refused before anything runs.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import synth
from fsdp2_layout_aware_b200 import tide as T
from synth import configs

from _gpu_helpers import f32_bits, grads_to_dev
from _groups import mini_wan

pytestmark = pytest.mark.gpu


def params_of(group):
    return [(s[0], int(np.prod(s[1:], dtype=np.int64)) if len(s) > 1 else 1) for s in group.shapes]


def noalloc(group, dev_grads, out, scale_mode=T.TIDE_SCALE_INV_WORLD, max_ctas=0):
    flat = [g for row in dev_grads for g in row]
    return T.tide_rs_reduce_noalloc(params_of(group), group.world, [g.data_ptr() for g in flat],
                                    [g.numel() for g in flat], out.data_ptr(), out.numel(),
                                    scale_mode, max_ctas,
                                    int(torch.cuda.current_stream().cuda_stream))


def with_plan(group, dev_grads, scale_mode):
    plan = T.Plan(group.shapes, group.world)
    out = torch.full((group.world * plan.shard_numel,), float("nan"), device="cuda")
    plan.rs_reduce(dev_grads, out, scale_mode=scale_mode)
    return out


def test_noalloc_matches_planned_reduce_on_consecutive_calls():
    a = configs.tiny()                   # W=4, misaligned chunks, pad rows
    b = mini_wan()                       # W=16, all-pad chunks, small chunks
    ga = grads_to_dev(a, synth.grads_host(a, seed=101))
    gb = grads_to_dev(b, synth.grads_host(b, seed=102))
    ga2 = grads_to_dev(a, synth.grads_host(a, seed=103))
    runs = [(a, ga, T.TIDE_SCALE_INV_WORLD), (b, gb, T.TIDE_SCALE_NONE),
            (a, ga2, T.TIDE_SCALE_INV_WORLD)]
    outs = []
    for group, grads, scale in runs:     # back to back on one stream, no sync in between
        n = group.world * T.Plan(group.shapes, group.world, host_only=True).shard_numel
        out = torch.full((n,), float("nan"), device="cuda")
        assert noalloc(group, grads, out, scale) == T.TIDE_OK
        outs.append(out)
    torch.cuda.synchronize()
    for (group, grads, scale), out in zip(runs, outs):
        ref = with_plan(group, grads, scale)
        torch.cuda.synchronize()
        assert np.array_equal(f32_bits(out), f32_bits(ref)), group.name


def test_noalloc_max_ctas_and_size_limit():
    g = configs.qwen3moe(4)
    grads = grads_to_dev(g, synth.grads_host(g, seed=104))
    n = g.world * T.Plan(g.shapes, g.world, host_only=True).shard_numel
    out8 = torch.empty(n, device="cuda")
    out_all = torch.empty(n, device="cuda")
    assert noalloc(g, grads, out8, max_ctas=8) == T.TIDE_OK
    assert noalloc(g, grads, out_all) == T.TIDE_OK
    ref = with_plan(g, grads, T.TIDE_SCALE_INV_WORLD)
    torch.cuda.synchronize()
    assert np.array_equal(f32_bits(out8), f32_bits(ref))
    assert np.array_equal(f32_bits(out_all), f32_bits(ref))
    # 600 params over 256 ranks need 600 * (32 + 8 * 256) bytes > 1 MiB: refused up front
    big = [(256, 1)] * 600
    assert 600 * (32 + 8 * 256) > T.TIDE_NOALLOC_SCRATCH_BYTES
    st = T.tide_rs_reduce_noalloc(big, 256, [0] * (600 * 256), [256] * (600 * 256),
                                  out_all.data_ptr(), out_all.numel(), 1, 0, 0)
    assert st == T.TIDE_ERR_SIZE
