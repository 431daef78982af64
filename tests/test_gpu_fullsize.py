"""GPU parity at the full workload sizes, in the launch configuration the benchmark times.

Inputs are generated on the device by the generator's CUDA twin; the oracle
side regenerates only the values it needs on the host.  Checked outputs: a
seeded random sample plus the first and last element of every chunk of every
rank (pad boundaries included) for RS, and the same for AG placement, each
compared bit for bit with the oracle's per-element answer.  This also checks
that the device generator reproduces the host generator.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from fsdp2_layout_aware_b200 import tide as T
from synth import configs

from _gpu_helpers import bits_of

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SEED = 1


def sample_positions(group, L, n_random, rng):
    """(rank, j) output positions: random ones plus both ends of every chunk and its valid part."""
    W, Ns = group.world, L.Ns
    pos = set()
    if Ns == 0:
        return []
    for r in range(W):
        for i in range(group.n_params):
            c = L.c[i]
            if c == 0:
                continue
            valid = max(0, min(c, group.numel(i) - r * c))
            for e in {0, c - 1, valid - 1, valid, c // 2}:
                if 0 <= e < c:
                    pos.add((r, L.off[i] + e))
    flat = rng.integers(0, W * Ns, size=n_random)
    pos.update((int(f // Ns), int(f % Ns)) for f in flat)
    return sorted(pos)


def rank_values(group, positions):
    """(located, vals): the oracle's locate() of each position and the W bf16 inputs there."""
    W = group.world
    zero = [synth.zero_grad_params(group, SEED, k) for k in range(W)]
    located = [oracle.locate(W, group.shapes, r, j) for r, j in positions]
    need = {}
    for n, (st, i, src) in enumerate(located):
        if st == 1:
            need.setdefault(i, []).append((n, src))
    vals = np.zeros((len(positions), W), dtype=np.uint16)
    for i, lst in need.items():
        idx = np.array([s for _, s in lst], dtype=np.int64)
        rows = np.array([n for n, _ in lst])
        for k in range(W):
            if i in zero[k]:
                continue
            vals[rows, k] = synth.gather_bf16(idx, SEED, synth.STREAM_GRAD, k, i, group.grad_sigma)
    return located, vals


def expected_rs(group, L, positions, scale):
    """Oracle value at each sampled output position, from host-regenerated inputs."""
    located, vals = rank_values(group, positions)
    out = np.zeros(len(positions), dtype=np.float32)
    for n, (st, _, _) in enumerate(located):
        out[n] = oracle.sum_ranks(vals[n], scale) if st == 1 else np.float32(0.0)
    return out


def check_rs(group, out, L, scale, rng, n_random=20000):
    pos = sample_positions(group, L, n_random, rng)
    flat = torch.tensor([r * L.Ns + j for r, j in pos], dtype=torch.int64, device=out.device)
    got = out[flat].cpu().numpy()
    exp = expected_rs(group, L, pos, scale)
    bad = np.nonzero(got.view(np.uint32) != exp.view(np.uint32))[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {pos[bad[0]]}: {got[bad[0]]} vs {exp[bad[0]]}"


def check_ag(group, params, L, rng, n_random=4000):
    W, Ns = group.world, L.Ns
    for i in range(group.n_params):
        c = L.c[i]
        if c == 0:
            continue
        qs = set(rng.integers(0, W * c, size=max(1, n_random // group.n_params)).tolist())
        for r in range(W):
            valid = max(0, min(c, group.numel(i) - r * c))
            for e in {0, c - 1, valid - 1, valid}:
                if 0 <= e < c:
                    qs.add(r * c + e)
        qs = sorted(qs)
        got = bits_of(params[i][torch.tensor(qs, dtype=torch.int64, device=params[i].device)])
        exp = np.zeros(len(qs), dtype=np.uint16)
        by_rank = {}
        for n, q in enumerate(qs):
            st, a = oracle.ag_source(W, group.shapes, i, q)
            if st == 1:
                by_rank.setdefault(a // Ns, []).append((n, a % Ns))
        for r, lst in by_rank.items():
            idx = np.array([j for _, j in lst], dtype=np.int64)
            exp[[n for n, _ in lst]] = synth.gather_bf16(idx, SEED, synth.STREAM_AG, r, 0,
                                                         group.param_sigma)
        assert np.array_equal(got, exp), f"param {i}"


FULL = ["llama70b", "qwen3moe", "wan14b"] + [f"sweep_w{w}" for w in configs.SWEEP_WORLDS]


@pytest.mark.parametrize("name", FULL)
def test_full_size_rs_and_ag(name):
    group = configs.by_name(name)
    rng = np.random.default_rng(7)
    torch.cuda.empty_cache()
    plan = T.Plan(group.shapes, group.world)
    L = oracle.layout(group.world, group.shapes)
    assert plan.shard_numel == L.Ns
    grads = synth.dev_grads(group, SEED)
    out = torch.full((group.world * L.Ns,), float("nan"), device="cuda")
    plan.rs_reduce(grads, out, scale_mode=T.TIDE_SCALE_INV_WORLD)     # the benchmark's call
    torch.cuda.synchronize()
    plan.check()
    check_rs(group, out, L, 1, rng)
    if name == "wan14b":
        # Slot-Reuse: stage into vacated all-gather slots, then reduce: must equal plain mode
        ref = out.clone()
        slots = [torch.empty(group.world * L.Ns, dtype=torch.bfloat16, device="cuda")
                 for _ in range(group.world)]
        for engine in (T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE):
            out.fill_(float("nan"))
            plan.rs_reduce(grads, out, scale_mode=T.TIDE_SCALE_INV_WORLD, slots=slots, engine=engine)
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
        del slots, ref
    del grads, out
    torch.cuda.empty_cache()
    ag = synth.dev_ag(group, L.Ns, SEED)
    params = [torch.full((group.world * L.c[i],), 0x7777, dtype=torch.int16, device="cuda")
              .view(torch.bfloat16) for i in range(group.n_params)]
    for engine in (T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE):
        plan.ag_place(ag, params, engine=engine)
        torch.cuda.synchronize()
        plan.check()
        check_ag(group, params, L, rng)
        for p in params:
            p.view(torch.int16).fill_(0x7777)
    del ag, params
    torch.cuda.empty_cache()


def bf16_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("name", ["llama70b", "qwen3moe", "wan14b"])
def test_full_size_other_modes(name):
    """At full size: tree order bit-exact against the oracle's tree (and within 1e-6 *
    sum|terms| of the exact sum) at sampled positions; the bulk-copy kernel and the
    pipelined Slot-Reuse (W segments, copy engines on a second stream) give the plain call's
    bits."""
    group = configs.by_name(name)
    W = group.world
    rng = np.random.default_rng(8)
    torch.cuda.empty_cache()
    plan = T.Plan(group.shapes, W)
    L = oracle.layout(W, group.shapes)
    grads = synth.dev_grads(group, SEED)
    n = W * L.Ns
    ref = torch.full((n,), float("nan"), device="cuda")
    plan.rs_reduce(grads, ref, scale_mode=T.TIDE_SCALE_INV_WORLD)
    torch.cuda.synchronize()
    check_rs(group, ref, L, 1, rng, n_random=5000)
    out = torch.full((n,), float("nan"), device="cuda")
    # tree order, unscaled: exact sums at sampled positions (W <= 64 bf16 terms: exact in fp64)
    plan.rs_reduce(grads, out, scale_mode=T.TIDE_SCALE_NONE, order=T.TIDE_ORDER_TREE)
    torch.cuda.synchronize()
    plan.check()
    assert plan.last_launch()[0] == T.K_RS_TREE_V32          # W = 8 or 16: the 32-byte tree kernel
    pos = sample_positions(group, L, 20000, rng)
    located, vals = rank_values(group, pos)
    terms = bf16_to_f64(vals)
    E, A = terms.sum(axis=1), np.abs(terms).sum(axis=1)
    flat = torch.tensor([r * L.Ns + j for r, j in pos], dtype=torch.int64, device="cuda")
    got32 = out[flat].cpu().numpy()
    got = got32.astype(np.float64)
    assert np.all(np.abs(got - E) <= 1e-6 * A)
    pads = np.array([st != 1 for st, _, _ in located])
    assert np.all(got[pads] == 0.0)
    want = np.array([oracle.sum_ranks_tree(vals[n], 0) if st == 1 else np.float32(0.0)
                     for n, (st, _, _) in enumerate(located)], dtype=np.float32)
    assert np.array_equal(got32.view(np.uint32), want.view(np.uint32))
    # the bulk-copy kernel
    tma = T.Plan(group.shapes, W, tma=True)
    out.fill_(float("nan"))
    tma.rs_reduce(grads, out, scale_mode=T.TIDE_SCALE_INV_WORLD)
    torch.cuda.synchronize()
    tma.check()
    assert tma.last_launch()[0] == T.K_RS_TMA
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
    tma.close()
    # pipelined Slot-Reuse, W segments
    slots = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    cs = torch.cuda.Stream()
    out.fill_(float("nan"))
    plan.rs_reduce_pipelined(grads, out, slots, W, cs)
    torch.cuda.synchronize()
    plan.check()
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32))
    del slots, grads, out, ref
    torch.cuda.empty_cache()


def test_device_generator_matches_host():
    g = configs.tiny()
    dev = synth.dev_grads(g, 5)
    host = synth.grads_host(g, 5)
    for k in range(g.world):
        for i in range(g.n_params):
            assert np.array_equal(bits_of(dev[k][i]), host[k][i])
    q = configs.qwen3moe(20)                      # one unrouted expert per rank
    assert q.n_zero_experts == 1
    devq = synth.dev_grads(q, 3)
    for k in range(q.world):
        zero = synth.zero_grad_params(q, 3, k)
        assert len(zero) == 3
        for i in sorted(zero | {0, 4, 7, q.n_params - 1}):
            h = synth.grad_host(q, 3, k, i)
            assert np.array_equal(bits_of(devq[k][i]), h)
            assert (i in zero) == (not h.any())


def test_a_param_beyond_2_to_the_31_elements():
    """One param of (2^21 + 3) x 1024 = 2,147,486,720 elements (more than 2^31) over W = 2: its
    chunk offsets, the fp32 shards' indices and the placement's destination indices pass 2^31,
    so any 32-bit element index would show.  Sampled outputs (chunk ends, the valid/pad
    boundary, random positions, and the positions around element 2^31 of the output and of
    the padded storage) against the oracle's answer for each position, RS and AG."""
    group = configs.Group("beyond_2_31", 2, ((2 ** 21 + 3, 1024), (5,)))
    rng = np.random.default_rng(11)
    torch.cuda.empty_cache()
    plan = T.Plan(group.shapes, group.world)
    L = oracle.layout(group.world, group.shapes)
    assert group.numel(0) > 2 ** 31 and 2 * L.Ns > 2 ** 31
    grads = synth.dev_grads(group, SEED)
    out = torch.full((2 * L.Ns,), float("nan"), device="cuda")
    plan.rs_reduce(grads, out, scale_mode=T.TIDE_SCALE_INV_WORLD)
    torch.cuda.synchronize()
    plan.check()
    check_rs(group, out, L, 1, rng, n_random=5000)
    pos = [(int(f // L.Ns), int(f % L.Ns)) for f in range(2 ** 31 - 40, 2 ** 31 + 40)]
    flat = torch.tensor([r * L.Ns + j for r, j in pos], dtype=torch.int64, device="cuda")
    got = out[flat].cpu().numpy()
    assert np.array_equal(got.view(np.uint32), expected_rs(group, L, pos, 1).view(np.uint32))
    del grads, out
    torch.cuda.empty_cache()
    ag = synth.dev_ag(group, L.Ns, SEED)
    params = [torch.full((2 * L.c[i],), 0x7777, dtype=torch.int16, device="cuda").view(torch.bfloat16)
              for i in range(group.n_params)]
    plan.ag_place(ag, params)
    torch.cuda.synchronize()
    plan.check()
    check_ag(group, params, L, rng, n_random=2000)
    qs = list(range(2 ** 31 - 40, 2 ** 31 + 40))
    got = bits_of(params[0][torch.tensor(qs, dtype=torch.int64, device="cuda")])
    exp = np.zeros(len(qs), dtype=np.uint16)
    for n, q in enumerate(qs):
        st, a = oracle.ag_source(2, group.shapes, 0, q)
        if st == 1:
            exp[n] = synth.gather_bf16(np.array([a % L.Ns], dtype=np.int64), SEED, synth.STREAM_AG,
                                       a // L.Ns, 0, group.param_sigma)[0]
    assert np.array_equal(got, exp)
    del ag, params
    torch.cuda.empty_cache()
