"""tide_rs_reduce_noalloc: the allocation-free reduction, through the C-ABI.

Some callers cannot allocate device memory (for example a runtime whose
caching allocator owns the GPU's memory), so they cannot build a plan, whose
tables tide_plan_group allocates.  tide_rs_reduce_noalloc keeps its tables in
a fixed 1 MiB device array instead.  These tests check that it returns the
same fp32 shards, bit for bit, as the CPU oracle and as tide_rs_reduce: on
groups called back to back (the shared array is rewritten between them), on
buffers at odd element offsets with guard bands, on a W=64 group, with a CTA
cap; that a group too large for the array is refused before anything runs; and
that a call on a stream being captured is refused.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from fsdp2_layout_aware_b200 import tide as T
from synth import configs

from _gpu_helpers import f32_bits, grads_to_dev, to_dev
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


def shard_numel(group):
    return group.world * T.Plan(group.shapes, group.world, host_only=True).shard_numel


def oracle_bits(group, grads_host, scale_mode):
    return oracle.rs_reduce(group.world, group.shapes, grads_host, scale_mode).view(np.uint32)


def test_noalloc_matches_oracle_and_plan_on_consecutive_calls():
    a = configs.tiny()                   # W=4, misaligned chunks, pad rows
    b = mini_wan()                       # W=16, all-pad chunks, small chunks
    ha, hb, ha2 = (synth.grads_host(a, seed=101), synth.grads_host(b, seed=102),
                   synth.grads_host(a, seed=103))
    runs = [(a, ha, T.TIDE_SCALE_INV_WORLD), (b, hb, T.TIDE_SCALE_NONE),
            (a, ha2, T.TIDE_SCALE_INV_WORLD)]
    dev = [grads_to_dev(g, h) for g, h, _ in runs]
    outs = []
    for (group, _, scale), grads in zip(runs, dev):   # back to back on one stream, no sync
        out = torch.full((shard_numel(group),), float("nan"), device="cuda")
        assert noalloc(group, grads, out, scale) == T.TIDE_OK
        outs.append(out)
    torch.cuda.synchronize()
    for (group, host, scale), grads, out in zip(runs, dev, outs):
        assert np.array_equal(f32_bits(out), oracle_bits(group, host, scale)), group.name
        ref = with_plan(group, grads, scale)
        torch.cuda.synchronize()
        assert np.array_equal(f32_bits(out), f32_bits(ref)), group.name


def test_noalloc_max_ctas_and_size_limit():
    g = configs.qwen3moe(4)
    host = synth.grads_host(g, seed=104)
    grads = grads_to_dev(g, host)
    n = shard_numel(g)
    out8 = torch.empty(n, device="cuda")
    out_all = torch.empty(n, device="cuda")
    assert noalloc(g, grads, out8, max_ctas=8) == T.TIDE_OK
    assert noalloc(g, grads, out_all) == T.TIDE_OK
    ref = with_plan(g, grads, T.TIDE_SCALE_INV_WORLD)
    torch.cuda.synchronize()
    want = oracle_bits(g, host, T.TIDE_SCALE_INV_WORLD)
    assert np.array_equal(f32_bits(out8), want)
    assert np.array_equal(f32_bits(out_all), want)
    assert np.array_equal(f32_bits(ref), want)
    # 600 params over 256 ranks need 600 * (32 + 8 * 256) bytes > 1 MiB: refused up front
    big = [(256, 1)] * 600
    assert 600 * (32 + 8 * 256) > T.TIDE_NOALLOC_SCRATCH_BYTES
    st = T.tide_rs_reduce_noalloc(big, 256, [0] * (600 * 256), [256] * (600 * 256),
                                  out_all.data_ptr(), out_all.numel(), 1, 0, 0)
    assert st == T.TIDE_ERR_SIZE


def test_noalloc_world_64():
    """W = 64 (rows < W, an exact multiple, a 1-D and a ragged param): 64 * 5 grads."""
    g = configs.Group("w64", 64, ((200, 24), (192, 16), (33,), (1000,), (7, 5)))
    assert 5 * (32 + 8 * 64) <= T.TIDE_NOALLOC_SCRATCH_BYTES
    host = synth.grads_host(g, seed=105)
    grads = grads_to_dev(g, host)
    for scale in (T.TIDE_SCALE_INV_WORLD, T.TIDE_SCALE_NONE):
        out = torch.full((shard_numel(g),), float("nan"), device="cuda")
        assert noalloc(g, grads, out, scale) == T.TIDE_OK
        torch.cuda.synchronize()
        assert np.array_equal(f32_bits(out), oracle_bits(g, host, scale))


@pytest.mark.parametrize("shift", [1, 3])
def test_noalloc_misaligned_buffers_and_guard_bands(shift):
    """Gradients and output at odd element offsets take the element-by-element path;
    the guard bands around every buffer stay untouched."""
    group = configs.Group("mis", 4, ((37, 16), (1000,), (129, 64)))
    host = synth.grads_host(group, seed=106)
    W, P = group.world, group.n_params
    guard = 64
    pool, dev = [], []
    for k in range(W):
        row = []
        for i in range(P):
            n = group.numel(i)
            buf = torch.full((n + shift + guard,), -3, dtype=torch.int16, device="cuda")
            buf[shift: shift + n] = to_dev(host[k][i]).view(torch.int16)
            pool.append(buf)
            row.append(buf[shift: shift + n].view(torch.bfloat16))
        dev.append(row)
    n_out = shard_numel(group)
    out_buf = torch.full((n_out + 2 * guard + shift,), 12345.0, device="cuda")
    out = out_buf[guard + shift: guard + shift + n_out]
    assert noalloc(group, dev, out) == T.TIDE_OK
    torch.cuda.synchronize()
    assert np.array_equal(f32_bits(out), oracle_bits(group, host, T.TIDE_SCALE_INV_WORLD))
    ob = out_buf.cpu().numpy()
    assert np.all(ob[: guard + shift] == 12345.0) and np.all(ob[guard + shift + n_out:] == 12345.0)
    for buf in pool:
        assert torch.all(buf[:shift] == -3) and torch.all(buf[-guard:] == -3)


@pytest.mark.filterwarnings("ignore:The CUDA Graph is empty")   # the refused call enqueued nothing
def test_noalloc_refuses_a_capturing_stream():
    """Its tables are copied from a host array the next call reuses, so a capture is refused
    with nothing enqueued; a later uncaptured call still gives the oracle's bits."""
    g = configs.tiny()
    host = synth.grads_host(g, seed=107)
    grads = grads_to_dev(g, host)
    out = torch.full((shard_numel(g),), float("nan"), device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        assert noalloc(g, grads, out) == T.TIDE_OK      # first call on the device: set-up
    torch.cuda.synchronize()
    out.fill_(float("nan"))
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    status = []
    with torch.cuda.graph(graph, stream=s):
        status.append(noalloc(g, grads, out))
    assert status == [T.TIDE_ERR_INVALID_ARG]
    del graph
    assert torch.isnan(out).all()
    with torch.cuda.stream(s):
        assert noalloc(g, grads, out) == T.TIDE_OK
    torch.cuda.synchronize()
    assert np.array_equal(f32_bits(out), oracle_bits(g, host, T.TIDE_SCALE_INV_WORLD))
