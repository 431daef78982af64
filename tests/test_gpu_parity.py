"""GPU parity: the CUDA path through the C-ABI against the CPU oracle, element by element.

Bars: AG placement, Slot-Reuse staging, rank-order RS and tree-order RS bit-exact
against the oracle (tree order also within 1e-6 * sum|terms| of the exact fp64 sum).  Sizes are small enough for
the oracle to finish in seconds but span many tiles, ragged tile ends,
misaligned chunk offsets, pad rows and all-pad chunks.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from fsdp2_layout_aware_b200 import tide as T
from synth import configs

from _gpu_helpers import bits_of, f32_bits, grads_to_dev, padded_params, poison_pads, to_dev
from _groups import degenerate, mini_sweep, mini_wan, random_group

pytestmark = pytest.mark.gpu


def parity_groups():
    rng = np.random.default_rng(2024)
    out = [configs.tiny(), degenerate(), mini_wan(), mini_sweep(2), mini_sweep(64),
           configs.qwen3moe(4), configs.Group("long_chunk", 3, ((30011, 7), (5,), (40000,)))]
    for w in (1, 2, 3, 5, 8, 16, 64):
        out.append(random_group(rng, w, int(rng.integers(1, 8)), max_rows=1500, name=f"rand_w{w}"))
    # W = 32: the tree order's compile-time four-group kernel
    out.append(random_group(np.random.default_rng(32), 32, 5, max_rows=1500, name="rand_w32"))
    return out


GROUPS = parity_groups()
IDS = [f"{g.name}_w{g.world}" for g in GROUPS]


def run_rs(group, grads_host, scale=1, order=0, max_ctas=0, slots=False, engine=0, tma=False,
           out_shift=0, short_ctas=False):
    """out_shift > 0 places the output that many floats past a 512-byte boundary (4: 16-byte but
    not 32-byte aligned, which rules out the 32-byte kernels)."""
    plan = T.Plan(group.shapes, group.world, tma=tma, short_ctas=short_ctas)
    grads = grads_to_dev(group, grads_host)
    n = group.world * plan.shard_numel
    out = torch.full((n + out_shift,), float("nan"), device="cuda")[out_shift:]
    slot_bufs = None
    if slots:
        slot_bufs = [torch.full((group.world * plan.shard_numel,), -1, dtype=torch.int16,
                                device="cuda").view(torch.bfloat16) for _ in range(group.world)]
    plan.rs_reduce(grads, out, scale_mode=scale, order=order, slots=slot_bufs, engine=engine,
                   max_ctas=max_ctas)
    torch.cuda.synchronize()
    plan.check()
    return out, slot_bufs, plan


@pytest.mark.parametrize("group", GROUPS, ids=IDS)
@pytest.mark.parametrize("scale", [0, 1])
@pytest.mark.parametrize("tma", [False, True], ids=["lsu", "tma"])
def test_rs_rank_order_bit_exact(group, scale, tma):
    grads = synth.grads_host(group, seed=31)
    out, _, plan = run_rs(group, grads, scale=scale, tma=tma)
    ref = oracle.rs_reduce(group.world, group.shapes, grads, scale)
    assert np.array_equal(f32_bits(out), ref.view(np.uint32))
    kernel, ctas = plan.last_launch()
    if plan.n_tiles:
        lsu = (T.K_RS, T.K_RS_V32)
        assert kernel in (lsu + (T.K_RS_TMA,) if tma else lsu) and ctas > 0


def aligned_group(world, seed):
    """Shapes whose chunks all start on 8-element boundaries (the bulk-copy path)."""
    rng = np.random.default_rng(seed)
    shapes = []
    for _ in range(int(rng.integers(2, 7))):
        d0 = int(rng.integers(1, 3000))
        shapes.append((d0, 8 * int(rng.integers(1, 40))))
    shapes.append((world * 8 * int(rng.integers(1, 50)),))
    return configs.Group(f"aligned_w{world}", world, tuple(shapes))


TMA_GROUPS = [aligned_group(w, w) for w in (1, 2, 3, 8, 16, 64, 256)] + [mini_sweep(8), configs.qwen3moe(4)]


@pytest.mark.parametrize("group", TMA_GROUPS, ids=[f"{g.name}_w{g.world}" for g in TMA_GROUPS])
def test_rs_bulk_copy_path(group):
    """The TMA reduction (opt-in): taken for aligned groups, bit-exact, any CTA count, both orders."""
    grads = synth.grads_host(group, seed=33)
    ref = oracle.rs_reduce(group.world, group.shapes, grads, 1)
    E, A = oracle.exact_f64(group.world, group.shapes, grads)
    for ctas in (1, 7, 0):
        out, _, plan = run_rs(group, grads, scale=1, max_ctas=ctas, tma=True)
        assert plan.last_launch()[0] == T.K_RS_TMA
        assert np.array_equal(f32_bits(out), ref.view(np.uint32)), f"max_ctas={ctas}"
    out, _, plan = run_rs(group, grads, scale=0, order=1, tma=True)
    assert plan.last_launch()[0] == T.K_RS_TMA
    assert np.all(np.abs(out.cpu().numpy().astype(np.float64) - E) <= 1e-6 * A)
    tree = oracle.rs_reduce_tree(group.world, group.shapes, grads, 0)
    assert np.array_equal(f32_bits(out), tree.view(np.uint32))
    for engine in (T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE):
        out, _, plan = run_rs(group, grads, scale=1, slots=True, engine=engine, tma=True)
        assert plan.last_launch()[0] == T.K_SLOT_RS_TMA
        assert np.array_equal(f32_bits(out), ref.view(np.uint32))


@pytest.mark.parametrize("seed", range(1, 17))
def test_rs_tiny_all_seeds(seed):
    g = configs.tiny()
    grads = synth.grads_host(g, seed=seed)
    out, _, _ = run_rs(g, grads, scale=1)
    assert np.array_equal(f32_bits(out), oracle.rs_reduce(g.world, g.shapes, grads, 1).view(np.uint32))


@pytest.mark.parametrize("group", GROUPS, ids=IDS)
def test_rs_tree_order_within_tolerance(group):
    grads = synth.grads_host(group, seed=32)
    out, _, plan = run_rs(group, grads, scale=0, order=1)
    if plan.n_tiles:   # a tree kernel, on the grid its own occupancy gives
        k, ctas = plan.last_launch()
        assert k in (T.K_RS_TREE, T.K_RS_TREE_V32) and ctas == plan.launch_ctas(k, 0)
        if k == T.K_RS_TREE_V32:
            assert group.world in (2, 4, 8, 16)
    assert np.array_equal(f32_bits(out),
                          oracle.rs_reduce_tree(group.world, group.shapes, grads, 0).view(np.uint32))
    E, A = oracle.exact_f64(group.world, group.shapes, grads)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - E) <= 1e-6 * A)
    L = oracle.layout(group.world, group.shapes)
    pad = np.ones(group.world * L.Ns, dtype=bool)
    ref = oracle.rs_reduce(group.world, group.shapes, grads, 0)
    pad[np.nonzero(A)[0]] = False
    assert np.all(f32_bits(out)[A == 0] == ref.view(np.uint32)[A == 0])   # zeros / pads agree bitwise


@pytest.mark.parametrize("group", GROUPS, ids=IDS)
def test_tree_order_kernels_agree_bitwise(group):
    """Every tree-order kernel adds in the same tree: pairwise by levels, an odd one carried.
    Load/store (groups of 2, 4 or 8 ranks merged pairwise; 16- or 32-byte loads), bulk-copy,
    Slot-Reuse on SMs or copy engines, and any CTA count give the same bits."""
    grads = synth.grads_host(group, seed=35)
    ref, _, _ = run_rs(group, grads, scale=1, order=1)
    ref = f32_bits(ref)
    assert np.array_equal(ref, oracle.rs_reduce_tree(group.world, group.shapes, grads, 1).view(np.uint32))
    for kw in (dict(max_ctas=3), dict(tma=True), dict(slots=True),
               dict(slots=True, engine=T.TIDE_ENGINE_CE), dict(out_shift=4)):
        out, _, plan = run_rs(group, grads, scale=1, order=1, **kw)
        assert np.array_equal(f32_bits(out), ref), kw
        if kw == dict(out_shift=4) and plan.n_tiles:
            assert plan.last_launch()[0] == T.K_RS_TREE     # the 16-byte tree kernel


@pytest.mark.parametrize("slots", [False, True], ids=["plain", "slot"])
def test_bulk_copy_wait_timeout_is_reported_and_recovered(slots):
    """A bounded wait that runs out.  Test hook: CTA 0 of the bulk-copy kernel withholds its
    first stage, so its consumers' wait gives up after about 1 s. The CTA then stops and waits
    for its own copies in flight. The launch reports TIDE_KCHECK_TIMEOUT in the error word,
    and the context stays usable."""
    group = aligned_group(8, 3)
    grads = synth.grads_host(group, seed=36)
    ref = oracle.rs_reduce(group.world, group.shapes, grads, 1)
    plan = T.Plan(group.shapes, group.world, tma=True, test_tma_timeout=True)
    assert plan.n_tiles > 0
    dev = grads_to_dev(group, grads)
    n = group.world * plan.shard_numel
    slot_bufs = ([torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(group.world)]
                 if slots else None)
    out = torch.full((n,), float("nan"), device="cuda")
    torch.cuda.synchronize()
    t0 = time.monotonic()
    plan.rs_reduce(dev, out, slots=slot_bufs)
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    assert plan.last_launch()[0] == (T.K_SLOT_RS_TMA if slots else T.K_RS_TMA)
    assert plan.errors() == T.TIDE_KCHECK_TIMEOUT
    assert plan.errors() == 0                       # read and cleared
    assert 0.5 < elapsed < 60
    # CTAs other than 0 finished their tiles: those outputs are the oracle's
    got = f32_bits(out)
    done = got == ref.view(np.uint32)
    assert done.mean() > 0.5
    # the context is intact: a plan without the hook gives the oracle's bits
    plan.close()
    out2, _, plan2 = run_rs(group, grads, scale=1, tma=True, slots=slots)
    assert plan2.last_launch()[0] == (T.K_SLOT_RS_TMA if slots else T.K_RS_TMA)
    assert np.array_equal(f32_bits(out2), ref.view(np.uint32))


@pytest.mark.parametrize("W", [2, 4, 8, 16, 64, 256])
def test_rs_identical_ranks_closed_form(W):
    """All ranks equal: unscaled sum is W*g exactly (any order), scaled is g."""
    g = configs.Group("ident", W, ((3 * W + 5, 17), (W // 2 + 1,)))
    one = synth.grads_host(configs.Group("src", 1, g.shapes), seed=5)[0]
    grads = [one for _ in range(W)]
    ref = oracle.pack_f32(W, g.shapes, one).astype(np.float64)
    for order in (0, 1):
        out, _, _ = run_rs(g, grads, scale=0, order=order)
        assert np.array_equal(out.cpu().numpy().astype(np.float64), W * ref)
        out, _, _ = run_rs(g, grads, scale=1, order=order)
        assert np.array_equal(out.cpu().numpy().astype(np.float64), ref)


def test_rs_rank_order_pin_on_gpu():
    # (1 + 2^-24) + 2^-24 = 1 in fp32 while 2^-24 + 2^-24 + 1 = 1 + 2^-23
    shapes = ((64,),)
    g = configs.Group("order", 3, shapes)
    def grads_of(vals):
        return [[np.full(64, np.array([v], np.float32).view(np.uint32)[0] >> 16, np.uint16)]
                for v in vals]
    for order, vals, exp in ((0, [1.0, 2.0 ** -24, 2.0 ** -24], 1.0),
                             (0, [2.0 ** -24, 2.0 ** -24, 1.0], 1.0 + 2.0 ** -23)):
        out, _, _ = run_rs(g, grads_of(vals), scale=0, order=order)
        L = oracle.layout(3, shapes)
        valid = out.cpu().numpy()[: L.c[0]]
        assert np.all(valid == np.float32(exp))


@pytest.mark.parametrize("vals,exp", [
    ([1.0, 2.0 ** -24, 2.0 ** -24, 2.0 ** -24], 1.0 + 2.0 ** -23),    # rank order gives 1
    ([1.0] + [2.0 ** -24] * 4, 1.0 + 2.0 ** -22),                       # a tie rounded to even
    ([1.0] + [2.0 ** -24] * 9, 1.0 + 2.0 ** -21),                       # W=10, two groups on the GPU
    ([1.0] + [2.0 ** -24] * 7, 1.0 + 3 * 2.0 ** -23),                   # W=8, 32-byte kernel
    ([1.0] + [2.0 ** -24] * 15, 1.0 + 7 * 2.0 ** -23),                  # W=16, 32-byte kernel
    ([1.0] + [2.0 ** -24] * 31, 1.0 + 15 * 2.0 ** -23),                 # W=32, four groups fixed
    ([1.0] + [2.0 ** -24] * 63, 1.0 + 31 * 2.0 ** -23),                 # W=64, eight groups fixed
])
def test_rs_tree_order_pin_on_gpu(vals, exp):
    """Worked values of the tree order (pairs by levels, odd one carried) on every tree kernel.
    W=8: [1, e, e, e, e, e, e, e] with e = 2^-24 gives (1+e) = 1 (tie to even), 2e, 2e, 2e;
    then 1 + 2^-23 and 2^-22; then 1 + 3*2^-23.  W=16, 32 and 64 likewise give 1 + 7*2^-23,
    1 + 15*2^-23 and 1 + 31*2^-23.  Rank order gives 1 for all of them."""
    W = len(vals)
    shapes = ((64 * W, 8),)
    g = configs.Group("tree_pin", W, shapes)
    grads = [[np.full(64 * W * 8, np.array([v], np.float32).view(np.uint32)[0] >> 16, np.uint16)]
             for v in vals]
    for kw in (dict(), dict(tma=True), dict(slots=True), dict(out_shift=4)):
        out, _, plan = run_rs(g, grads, scale=0, order=1, **kw)
        assert np.all(out.cpu().numpy() == np.float32(exp)), kw
        if not kw and W in (4, 8, 16):
            assert plan.last_launch()[0] == T.K_RS_TREE_V32


@pytest.mark.parametrize("group", GROUPS, ids=IDS)
@pytest.mark.parametrize("engine", [T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE])
def test_ag_place_bit_exact(group, engine):
    plan = T.Plan(group.shapes, group.world)
    L = oracle.layout(group.world, group.shapes)
    ag_bits = poison_pads(synth.ag_host(group, L.Ns, seed=41).reshape(-1), group, L)
    ag = to_dev(ag_bits)
    params = padded_params(plan, group)
    plan.ag_place(ag, params, engine=engine)
    torch.cuda.synchronize()
    plan.check()
    ref = oracle.ag_copyout(group.world, group.shapes, ag_bits)
    for p, r in zip(params, ref):
        assert np.array_equal(bits_of(p), r)


@pytest.mark.parametrize("group", [configs.tiny(), degenerate(), mini_wan(), configs.qwen3moe(4),
                                   GROUPS[-3]], ids=lambda g: f"{g.name}_w{g.world}")
@pytest.mark.parametrize("engine", [T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE])
def test_slot_reuse_equals_plain_and_oracle(group, engine):
    grads = synth.grads_host(group, seed=51)
    out, slots, plan = run_rs(group, grads, scale=1, slots=True, engine=engine)
    ref = oracle.rs_reduce(group.world, group.shapes, grads, 1)
    assert np.array_equal(f32_bits(out), ref.view(np.uint32))
    L = oracle.layout(group.world, group.shapes)
    for k in range(group.world):
        exp = np.full(group.world * L.Ns, 0xFFFF, dtype=np.uint16)   # slots started as -1 (0xFFFF)
        oracle.slot_stage(group.world, group.shapes, grads[k], exp)
        assert np.array_equal(bits_of(slots[k]), exp)


ONE_GROUPS = [configs.tiny(), degenerate(), mini_wan(), configs.qwen3moe(4), GROUPS[-3],
              aligned_group(8, 62)]


@pytest.mark.parametrize("group", ONE_GROUPS, ids=[f"{g.name}_w{g.world}" for g in ONE_GROUPS])
@pytest.mark.parametrize("engine", [T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE])
def test_each_rank_stages_its_own_slot_and_reduces_its_shard(group, engine):
    """Slot-Reuse as ranks that are processes run it: rank k stages only its own gradients into
    its own slot (tide_rs_stage_one), then rank r's one-rank plan reduces its shard from rows r
    of all W slots (tide_rs_reduce_slots).  Slot pads start as 0xFFFF (a bf16 NaN), so a read of
    a pad would show.  Each slot equals the oracle's staging of that rank, and each shard the
    oracle's rows r, in rank and in tree order."""
    W = group.world
    grads = synth.grads_host(group, seed=61)
    dev = grads_to_dev(group, grads)
    plan = T.Plan(group.shapes, W)
    L = oracle.layout(W, group.shapes)
    slots = [torch.full((W * L.Ns,), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
             for _ in range(W)]
    for k in range(W):
        plan.rs_stage_one(dev[k], slots[k], engine=engine)
    torch.cuda.synchronize()
    plan.check()
    for k in range(W):
        exp = np.full(W * L.Ns, 0xFFFF, dtype=np.uint16)
        oracle.slot_stage(W, group.shapes, grads[k], exp)
        assert np.array_equal(bits_of(slots[k]), exp), k
    for order, ref in ((T.TIDE_ORDER_RANK, oracle.rs_reduce(W, group.shapes, grads, 1)),
                       (T.TIDE_ORDER_TREE, oracle.rs_reduce_tree(W, group.shapes, grads, 1))):
        ref = ref.reshape(W, L.Ns)
        for r in range(W):
            mine = T.Plan(group.shapes, W, rank=r)
            out = torch.full((L.Ns,), float("nan"), device="cuda")
            mine.rs_reduce_slots(slots, out, scale_mode=T.TIDE_SCALE_INV_WORLD, order=order)
            torch.cuda.synchronize()
            mine.check()
            assert np.array_equal(f32_bits(out), ref[r].view(np.uint32)), (order, r)


V32_GROUPS = [aligned_group(w, 40 + w) for w in (2, 5, 8, 13, 16, 24, 32, 64)] + [configs.qwen3moe(4)]


@pytest.mark.parametrize("group", V32_GROUPS, ids=[f"{g.name}_w{g.world}" for g in V32_GROUPS])
def test_rs_32_byte_path(group):
    """W = 2 or W >= 5 with 32-byte aligned tiles takes the 32-byte variant; same bits."""
    grads = synth.grads_host(group, seed=34)
    L = oracle.layout(group.world, group.shapes)
    aligned16 = all((r * c) % 16 == 0 and (r * L.Ns + o) % 16 == 0
                    for c, o in zip(L.c, L.off) for r in range(group.world))
    for scale in (0, 1):
        ref = oracle.rs_reduce(group.world, group.shapes, grads, scale)
        for ctas in (0, 5):
            out, _, plan = run_rs(group, grads, scale=scale, max_ctas=ctas)
            assert plan.last_launch()[0] == (T.K_RS_V32 if aligned16 else T.K_RS)
            assert np.array_equal(f32_bits(out), ref.view(np.uint32))
        out, slots, plan = run_rs(group, grads, scale=scale, slots=True)
        assert plan.last_launch()[0] == (T.K_SLOT_RS_V32 if aligned16 else T.K_SLOT_RS)
        assert np.array_equal(f32_bits(out), ref.view(np.uint32))
    E, A = oracle.exact_f64(group.world, group.shapes, grads)
    out, _, _ = run_rs(group, grads, scale=0, order=1)
    assert np.all(np.abs(out.cpu().numpy().astype(np.float64) - E) <= 1e-6 * A)
    assert np.array_equal(f32_bits(out),
                          oracle.rs_reduce_tree(group.world, group.shapes, grads, 0).view(np.uint32))


def test_rs_32_byte_path_needs_32_byte_pointers():
    """Gradients 16- but not 32-byte aligned fall back to the 16-byte kernel, same bits."""
    group = mini_sweep(8)                                # tiles on 16-element boundaries
    grads = synth.grads_host(group, seed=35)
    plan = T.Plan(group.shapes, group.world)
    keep, dev = [], []
    for k in range(group.world):
        row = []
        for i in range(group.n_params):
            n = group.numel(i)
            buf = torch.empty(n + 8, dtype=torch.int16, device="cuda")
            buf[8:] = to_dev(grads[k][i]).view(torch.int16)
            keep.append(buf)
            row.append(buf[8:].view(torch.bfloat16))          # 16-byte offset
        dev.append(row)
    out = torch.empty(group.world * plan.shard_numel, device="cuda")
    plan.rs_reduce(dev, out)
    torch.cuda.synchronize()
    assert plan.last_launch()[0] == T.K_RS
    assert np.array_equal(f32_bits(out), oracle.rs_reduce(8, group.shapes, grads, 1).view(np.uint32))


# pad_tail: with 4 segments, the cut by valid elements leaves two groups empty
# and a last group of all-pad chunks and empty params (nothing to stage).
PIPE_GROUPS = [configs.tiny(), degenerate(), mini_wan(), configs.qwen3moe(4), aligned_group(16, 5),
               configs.Group("pad_tail", 4, ((8, 4), (1, 1000), (0, 3)))]


@pytest.mark.parametrize("group", PIPE_GROUPS, ids=[f"{g.name}_w{g.world}" for g in PIPE_GROUPS])
@pytest.mark.parametrize("segments", ["one", "three", "all"])
def test_slot_reuse_pipelined(group, segments):
    """Copy-engine staging on a second stream overlapped with the reduction: same bits."""
    n_seg = {"one": 1, "three": min(3, group.world), "all": group.world}[segments]
    grads = synth.grads_host(group, seed=53)
    ref = oracle.rs_reduce(group.world, group.shapes, grads, 1)
    L = oracle.layout(group.world, group.shapes)
    for tma, same_stream in ((False, False), (True, False), (False, True)):
        plan = T.Plan(group.shapes, group.world, tma=tma)
        dev = grads_to_dev(group, grads)
        n = group.world * plan.shard_numel
        slots = [torch.full((n,), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
                 for _ in range(group.world)]
        out = torch.full((n,), float("nan"), device="cuda")
        main = torch.cuda.current_stream()
        cs = main if same_stream else torch.cuda.Stream()
        plan.rs_reduce_pipelined(dev, out, slots, n_seg, cs)
        torch.cuda.synchronize()
        plan.check()
        assert np.array_equal(f32_bits(out), ref.view(np.uint32)), (tma, same_stream)
        for k in range(group.world):
            exp = np.full(n, 0xFFFF, dtype=np.uint16)
            oracle.slot_stage(group.world, group.shapes, grads[k], exp)
            assert np.array_equal(bits_of(slots[k]), exp)


@pytest.mark.parametrize("group", PIPE_GROUPS, ids=[f"{g.name}_w{g.world}" for g in PIPE_GROUPS])
def test_one_rank_pipelined_pulls_its_rows_on_the_copy_engines(group):
    """A one-rank plan's pipelined Slot-Reuse: the copy engines pull row r of every rank's
    gradients into W compact slots, the SMs reduce them segment by segment.  Each rank's shard
    equals the oracle's rows r (rank order, and tree order against the tree oracle), and each
    slot holds the oracle's staging of that rank restricted to row r (its pads untouched)."""
    W = group.world
    grads = synth.grads_host(group, seed=57)
    L = oracle.layout(W, group.shapes)
    refs = {T.TIDE_ORDER_RANK: oracle.rs_reduce(W, group.shapes, grads, 1).reshape(W, L.Ns),
            T.TIDE_ORDER_TREE: oracle.rs_reduce_tree(W, group.shapes, grads, 1).reshape(W, L.Ns)}
    staged = []
    for k in range(W):
        exp = np.full(W * L.Ns, 0xFFFF, dtype=np.uint16)
        oracle.slot_stage(W, group.shapes, grads[k], exp)
        staged.append(exp.reshape(W, L.Ns))
    dev = grads_to_dev(group, grads)
    cs = torch.cuda.Stream()
    for r in range(W):
        plan = T.Plan(group.shapes, W, rank=r)
        for order in (T.TIDE_ORDER_RANK, T.TIDE_ORDER_TREE):
            for n_seg in sorted({1, min(3, W), W}):
                rows = [torch.full((L.Ns,), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
                        for _ in range(W)]
                out = torch.full((L.Ns,), float("nan"), device="cuda")
                plan.rs_reduce_pipelined(dev, out, rows, n_seg, cs, order=order)
                torch.cuda.synchronize()
                plan.check()
                assert np.array_equal(f32_bits(out), refs[order][r].view(np.uint32)), (r, order, n_seg)
                for k in range(W):
                    assert np.array_equal(bits_of(rows[k]), staged[k][r]), (r, k, n_seg)


def test_slot_phases_separately():
    group = mini_wan()
    grads = synth.grads_host(group, seed=52)
    plan = T.Plan(group.shapes, group.world)
    dev = grads_to_dev(group, grads)
    n = group.world * plan.shard_numel
    slots = [torch.zeros(n, dtype=torch.bfloat16, device="cuda") for _ in range(group.world)]
    plan.rs_stage(dev, slots, engine=T.TIDE_ENGINE_SM)
    out = torch.empty(n, device="cuda")
    for order in (0, 1):
        plan.rs_reduce_slots(slots, out, scale_mode=0, order=order)
        torch.cuda.synchronize()
        assert plan.last_launch()[0] == (T.K_SLOT_RS_TREE if order else T.K_SLOT_RS)
        if order == 0:
            assert np.array_equal(f32_bits(out),
                                  oracle.rs_reduce(group.world, group.shapes, grads, 0).view(np.uint32))
        else:
            tree = oracle.rs_reduce_tree(group.world, group.shapes, grads, 0)
            assert np.array_equal(f32_bits(out), tree.view(np.uint32))


@pytest.mark.parametrize("group", [configs.tiny(), mini_sweep(8), configs.qwen3moe(4)],
                         ids=lambda g: g.name)
def test_max_ctas_does_not_change_bits(group):
    grads = synth.grads_host(group, seed=61)
    L = oracle.layout(group.world, group.shapes)
    ag_bits = synth.ag_host(group, L.Ns, seed=62).reshape(-1)
    ref_rs, ref_ag = None, None
    for ctas in (1, 8, 16, 32, 0):
        out, _, plan = run_rs(group, grads, scale=1, max_ctas=ctas)
        params = padded_params(plan, group)
        plan.ag_place(to_dev(ag_bits), params, max_ctas=ctas)
        torch.cuda.synchronize()
        rs_bits = f32_bits(out)
        ag_b = [bits_of(p) for p in params]
        if ref_rs is None:
            ref_rs, ref_ag = rs_bits, ag_b
        assert np.array_equal(rs_bits, ref_rs)
        for a, b in zip(ag_b, ref_ag):
            assert np.array_equal(a, b)
        if ctas:
            assert plan.launch_ctas(T.K_RS, ctas) == min(ctas, plan.n_tiles)


@pytest.mark.parametrize("shift", [1, 3, 8])
def test_misaligned_buffers_and_guard_bands(shift):
    """Buffers at 2-byte (not 16-byte) offsets take the scalar path; guards stay intact."""
    group = configs.Group("mis", 4, ((37, 16), (1000,), (129, 64)))
    grads = synth.grads_host(group, seed=71)
    plan = T.Plan(group.shapes, group.world)
    W, P, Ns = group.world, group.n_params, plan.shard_numel
    guard = 64
    pool = []
    dev = []
    for k in range(W):
        row = []
        for i in range(P):
            n = group.numel(i)
            buf = torch.full((n + shift + guard,), -3, dtype=torch.int16, device="cuda")
            buf[shift: shift + n] = to_dev(grads[k][i]).view(torch.int16)
            pool.append(buf)
            row.append(buf[shift: shift + n].view(torch.bfloat16))
        dev.append(row)
    out_buf = torch.full((W * Ns + 2 * guard + shift,), 12345.0, device="cuda")
    out = out_buf[guard + shift: guard + shift + W * Ns]
    plan.rs_reduce(dev, out, scale_mode=1)
    torch.cuda.synchronize()
    ref = oracle.rs_reduce(W, group.shapes, grads, 1)
    assert np.array_equal(f32_bits(out), ref.view(np.uint32))
    ob = out_buf.cpu().numpy()
    assert np.all(ob[: guard + shift] == 12345.0) and np.all(ob[guard + shift + W * Ns:] == 12345.0)
    for buf in pool:          # inputs untouched
        assert torch.all(buf[:shift] == -3) and torch.all(buf[-guard:] == -3)
    # AG into misaligned parameter storage with guards
    L = oracle.layout(W, group.shapes)
    ag_bits = synth.ag_host(group, L.Ns, seed=72).reshape(-1)
    ag_buf = torch.zeros(W * Ns + shift, dtype=torch.int16, device="cuda")
    ag_buf[shift:] = to_dev(ag_bits).view(torch.int16)
    bufs, params = [], []
    for i in range(P):
        n = W * L.c[i]
        b = torch.full((n + shift + guard,), 0x5555, dtype=torch.int16, device="cuda")
        bufs.append(b)
        params.append(b[shift: shift + n].view(torch.bfloat16))
    for engine in (T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE):
        plan.ag_place(ag_buf[shift:].view(torch.bfloat16), params, engine=engine)
        torch.cuda.synchronize()
        refp = oracle.ag_copyout(W, group.shapes, ag_bits)
        for b, p, r in zip(bufs, params, refp):
            assert np.array_equal(bits_of(p), r)
            assert torch.all(b[:shift] == 0x5555) and torch.all(b[-guard:] == 0x5555)


def test_guard_bands_aligned_fast_path():
    group = mini_sweep(8)
    grads = synth.grads_host(group, seed=73)
    plan = T.Plan(group.shapes, group.world)
    n = group.world * plan.shard_numel
    guard = 4096
    out_buf = torch.full((n + 2 * guard,), -7.0, device="cuda")
    out = out_buf[guard: guard + n]
    plan.rs_reduce(grads_to_dev(group, grads), out, scale_mode=1)
    torch.cuda.synchronize()
    assert np.array_equal(f32_bits(out), oracle.rs_reduce(8, group.shapes, grads, 1).view(np.uint32))
    assert torch.all(out_buf[:guard] == -7.0) and torch.all(out_buf[guard + n:] == -7.0)


def test_pointer_table_changes_between_calls():
    group = configs.tiny()
    plan = T.Plan(group.shapes, group.world)
    n = group.world * plan.shard_numel
    outs = []
    seeds = (81, 82, 81)
    keep = []
    for s in seeds:
        g = synth.grads_host(group, seed=s)
        dev = grads_to_dev(group, g)
        keep.append(dev)                       # distinct buffers each call
        out = torch.empty(n, device="cuda")
        plan.rs_reduce(dev, out, scale_mode=1)
        outs.append((out, g))
    torch.cuda.synchronize()
    for out, g in outs:
        assert np.array_equal(f32_bits(out), oracle.rs_reduce(4, group.shapes, g, 1).view(np.uint32))


def test_side_stream_and_empty_groups():
    group = configs.tiny()
    grads = synth.grads_host(group, seed=91)
    plan = T.Plan(group.shapes, group.world)
    s = torch.cuda.Stream()
    dev = grads_to_dev(group, grads)
    torch.cuda.synchronize()
    out = torch.empty(group.world * plan.shard_numel, device="cuda")
    with torch.cuda.stream(s):
        plan.rs_reduce(dev, out, scale_mode=1, stream=s)
    s.synchronize()
    assert np.array_equal(f32_bits(out), oracle.rs_reduce(4, group.shapes, grads, 1).view(np.uint32))
    # a group with no elements: every call is a no-op that succeeds
    empty = configs.Group("empty", 4, ((0,), (0, 9), (7, 0)))
    ep = T.Plan(empty.shapes, 4)
    z = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    ep.rs_reduce([[z, z, z] for _ in range(4)], torch.empty(0, device="cuda"))
    ep.ag_place(z, [z, z, z])
    ep.ag_place(z, [z, z, z], engine=T.TIDE_ENGINE_CE)
    torch.cuda.synchronize()
    ep.check()


@pytest.mark.parametrize("group", [configs.tiny(), mini_sweep(8)], ids=lambda g: g.name)
def test_cuda_graph_capture_and_replay(group):
    """After one uncaptured call with the same buffers (pointer tables on the device), the
    calls capture into a CUDA graph; replays read the buffers' current contents."""
    W = group.world
    plan = T.Plan(group.shapes, W)
    L = oracle.layout(W, group.shapes)
    n = W * plan.shard_numel
    dev = grads_to_dev(group, synth.grads_host(group, seed=94))
    out = torch.empty(n, device="cuda")
    out_pipe = torch.empty(n, device="cuda")
    slots = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    ag = to_dev(synth.ag_host(group, L.Ns, seed=95).reshape(-1))
    params = padded_params(plan, group)
    params_ce = padded_params(plan, group)
    cs = torch.cuda.Stream()
    side = torch.cuda.Stream()

    def step(stream):
        plan.ag_place(ag, params, stream=stream)
        # (uncaptured, the copy-engine call records and replays its own graph; inside the
        # capture it issues its copies into the caller's capture)
        plan.ag_place(ag, params_ce, engine=T.TIDE_ENGINE_CE, stream=stream)
        plan.rs_reduce(dev, out, stream=stream)
        plan.rs_reduce_pipelined(dev, out_pipe, slots, min(2, W), cs, stream=stream)

    with torch.cuda.stream(side):
        step(side)                                   # uploads the pointer tables
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(side)
    for seed in (96, 97):
        grads = synth.grads_host(group, seed=seed)
        ag_bits = synth.ag_host(group, L.Ns, seed=seed).reshape(-1)
        for k in range(W):
            for i in range(group.n_params):
                dev[k][i].copy_(to_dev(grads[k][i], group.shapes[i]))
        ag.copy_(to_dev(ag_bits))
        out.fill_(float("nan"))
        out_pipe.fill_(float("nan"))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        ref = oracle.rs_reduce(W, group.shapes, grads, 1).view(np.uint32)
        assert np.array_equal(f32_bits(out), ref)
        assert np.array_equal(f32_bits(out_pipe), ref)
        for p, pc, r in zip(params, params_ce, oracle.ag_copyout(W, group.shapes, ag_bits)):
            assert np.array_equal(bits_of(p), r)
            assert np.array_equal(bits_of(pc), r)
    plan.check()


@pytest.mark.filterwarnings("ignore:Warning. Profiler clears events")
def test_copy_engine_paths_launch_no_kernel():
    """AG placement and Slot-Reuse staging on the copy engines use no SM: the CUDA
    activity trace of those calls holds memcpy/memset records and no kernel."""
    from torch.profiler import ProfilerActivity, profile
    group = configs.tiny()
    W = group.world
    plan = T.Plan(group.shapes, W)
    L = oracle.layout(W, group.shapes)
    ag = to_dev(synth.ag_host(group, L.Ns, seed=98).reshape(-1))
    params = padded_params(plan, group)
    dev = grads_to_dev(group, synth.grads_host(group, seed=99))
    slots = [torch.empty(W * L.Ns, dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        plan.ag_place(ag, params, engine=T.TIDE_ENGINE_CE)
        plan.rs_stage(dev, slots, engine=T.TIDE_ENGINE_CE)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    assert names, "no CUDA activity recorded"
    assert all(("emcpy" in n) or ("emset" in n) for n in names), names
    assert plan.last_launch()[0] == -1
    # and the SM engine really launches kernels (the trace would show them)
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        plan.ag_place(ag, params, engine=T.TIDE_ENGINE_SM)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    assert any("ag_place_kernel" in n for n in names), names


def test_wrong_device_index_rejected():
    group = configs.tiny()
    st, h = T.tide_plan_group([(s[0], int(np.prod(s[1:]))) for s in group.shapes], 4,
                              torch.cuda.device_count(), 0)
    assert st in (T.TIDE_ERR_DEVICE, T.TIDE_ERR_CUDA) and h is None
    # the failed call leaves no stale runtime error behind: the next launch succeeds
    grads = synth.grads_host(group, seed=92)
    out, _, _ = run_rs(group, grads, scale=1)
    assert np.array_equal(f32_bits(out), oracle.rs_reduce(4, group.shapes, grads, 1).view(np.uint32))


def test_workspace_is_tables_only():
    for name in ("tiny", "wan14b"):
        g = configs.by_name(name)
        plan = T.Plan(g.shapes, g.world)
        W, P = g.world, g.n_params
        # tiles, numel table, error word, the reduction's two tile-claim counters, pointer
        # tables: grads, params, slots, shards
        expect = plan.n_tiles * 32 + 2 * P * 8 + 4 + 2 * 8 + W * P * 8 + P * 8 + W * 8 + W * 8
        assert plan.workspace_bytes == expect


@pytest.mark.parametrize("group", [configs.tiny(), mini_wan(), mini_sweep(8), configs.qwen3moe(4),
                                   degenerate()], ids=lambda g: f"{g.name}_w{g.world}")
def test_short_lived_ctas_give_the_same_bits(group):
    """TIDE_PLAN_SHORT_CTAS: one CTA per tile (per tile and rank when staging) that does its
    unit and exits.  Rank and tree order, Slot-Reuse on both engines and AG placement give the
    oracle's bits, with as many CTAs as units."""
    grads = synth.grads_host(group, seed=91)
    W = group.world
    ref = oracle.rs_reduce(W, group.shapes, grads, 1).view(np.uint32)
    out, _, plan = run_rs(group, grads, scale=1, short_ctas=True)
    assert np.array_equal(f32_bits(out), ref)
    if plan.n_tiles:
        assert plan.last_launch()[1] == plan.n_tiles
    out, _, _ = run_rs(group, grads, scale=1, order=1, short_ctas=True)
    assert np.array_equal(f32_bits(out), oracle.rs_reduce_tree(W, group.shapes, grads, 1).view(np.uint32))
    for engine in (T.TIDE_ENGINE_SM, T.TIDE_ENGINE_CE):
        out, _, plan = run_rs(group, grads, scale=1, slots=True, engine=engine, short_ctas=True)
        assert np.array_equal(f32_bits(out), ref)
    L = oracle.layout(W, group.shapes)
    ag_bits = poison_pads(synth.ag_host(group, L.Ns, seed=92).reshape(-1), group, L)
    params = padded_params(plan, group)
    plan.ag_place(to_dev(ag_bits), params)
    torch.cuda.synchronize()
    plan.check()
    for p, r in zip(params, oracle.ag_copyout(W, group.shapes, ag_bits)):
        assert np.array_equal(bits_of(p), r)
    if plan.n_tiles:
        assert plan.last_launch()[1] == plan.n_tiles
        assert plan.launch_ctas(T.K_STAGE, 0) == plan.n_tiles * W


@pytest.mark.parametrize("group", [configs.tiny(), mini_wan(), configs.qwen3moe(4)],
                         ids=lambda g: f"{g.name}_w{g.world}")
def test_copy_engine_calls_replay_recorded_graphs(group):
    """A copy-engine placement records its copies as a graph the first time a set of buffers
    is used and replays it when the same buffers come back.  Placement and gather placement
    give the oracle's bits on the recording call, on replays (outputs poisoned in between),
    with a second set of buffers, and back on the first; Slot-Reuse staging (issued
    directly) likewise on repeated calls."""
    W = group.world
    L = oracle.layout(W, group.shapes)
    plan = T.Plan(group.shapes, W)
    ag_bits = poison_pads(synth.ag_host(group, L.Ns, seed=93).reshape(-1), group, L)
    ag = to_dev(ag_bits)
    ref = oracle.ag_copyout(W, group.shapes, ag_bits)
    sets = [padded_params(plan, group), padded_params(plan, group)]
    rows = ag_bits.reshape(W, L.Ns)
    shards = [to_dev(rows[r]) for r in range(W)]
    for params in (sets[0], sets[0], sets[1], sets[0]):
        for fn in (lambda p: plan.ag_place(ag, p, engine=T.TIDE_ENGINE_CE),
                   lambda p: plan.ag_gather_place(shards, p, engine=T.TIDE_ENGINE_CE)):
            for t in params:
                t.view(torch.int16).fill_(0x7777)
            fn(params)
            torch.cuda.synchronize()
            for t, r in zip(params, ref):
                assert np.array_equal(bits_of(t), r)
    grads = synth.grads_host(group, seed=94)
    dev = grads_to_dev(group, grads)
    n = W * L.Ns
    slot_sets = [[torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(W)] for _ in range(2)]
    for slots in (slot_sets[0], slot_sets[0], slot_sets[1], slot_sets[0]):
        for sl in slots:
            sl.view(torch.int16).fill_(-1)
        plan.rs_stage(dev, slots, engine=T.TIDE_ENGINE_CE)
        torch.cuda.synchronize()
        for k in range(W):
            exp = np.full(n, 0xFFFF, dtype=np.uint16)
            oracle.slot_stage(W, group.shapes, grads[k], exp)
            assert np.array_equal(bits_of(slots[k]), exp)
    plan.check()


def test_tile_claims_on_long_launches_repeat_and_mix_with_fixed_strides():
    """Launches with 2+ CTAs per SM and 16+ tiles per CTA claim tiles from the plan's counters,
    and the launch's last CTA puts them back to zero.  Back-to-back launches on one plan
    (claiming, claiming, a capped fixed-stride launch, claiming, Slot-Reuse) each give the
    oracle's bits, so no launch inherits another's claims."""
    group = configs.Group("claims", 8, tuple((1024, 4096) for _ in range(16)))
    grads = synth.grads_host(group, seed=63)
    ref = oracle.rs_reduce(8, group.shapes, grads, 1).view(np.uint32)
    plan = T.Plan(group.shapes, 8)
    assert plan.n_tiles >= 16 * plan.launch_ctas(T.K_RS_V32, 0)
    dev = grads_to_dev(group, grads)
    n = 8 * plan.shard_numel
    for cap in (0, 0, 7, 0):
        out = torch.full((n,), float("nan"), device="cuda")
        plan.rs_reduce(dev, out, max_ctas=cap)
        torch.cuda.synchronize()
        plan.check()
        assert np.array_equal(f32_bits(out), ref), cap
    slots = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(8)]
    out = torch.full((n,), float("nan"), device="cuda")
    plan.rs_reduce(dev, out, slots=slots)
    torch.cuda.synchronize()
    assert np.array_equal(f32_bits(out), ref)
    # two plans claim from their own counters: their launches may run at the same time
    other = T.Plan(group.shapes, 8)
    outs = [torch.full((n,), float("nan"), device="cuda") for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    for _ in range(2):
        for pl, o, st in zip((plan, other), outs, streams):
            pl.rs_reduce(dev, o, stream=st)
    torch.cuda.synchronize()
    for o in outs:
        assert np.array_equal(f32_bits(o), ref)


@pytest.mark.parametrize("world", [128, 256])
def test_widest_groups_both_orders(world):
    """W = 128 and 256 (the library's limit): rank order on the 32-byte kernel, tree order on
    the run-time merge-stack kernel, both against the oracle; a ragged param and a param with
    fewer rows than ranks included."""
    group = configs.Group(f"wide_w{world}", world,
                          ((world * 24, 32), (world * 3 + 5, 16), (7, 48), (world * 48,)))
    grads = synth.grads_host(group, seed=67)
    for order, fn, kernel in ((0, oracle.rs_reduce, T.K_RS_V32), (1, oracle.rs_reduce_tree, T.K_RS_TREE)):
        ref = fn(world, group.shapes, grads, 1)
        out, _, plan = run_rs(group, grads, scale=1, order=order)
        assert plan.last_launch()[0] == kernel
        assert np.array_equal(f32_bits(out), ref.view(np.uint32)), order
    E, A = oracle.exact_f64(world, group.shapes, grads)
    out, _, _ = run_rs(group, grads, scale=0, order=1)
    assert np.all(np.abs(out.cpu().numpy().astype(np.float64) - E) <= 1e-6 * A)
