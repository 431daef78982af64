"""Pins for the CPU oracle: each check is fixed by something other than the oracle.

  * hand-derived layouts and a hand-worked two-rank example (tests/golden/);
  * torch.chunk + pad + cat (FSDP2's own dim-0 chunking) for the rank-major layout;
  * torch.distributed reduce_scatter_tensor over gloo for the reduce-scatter itself;
  * closed forms: identical ranks give W*g, one-hot ranks give g_k, small
    integers give exact sums (int64 brute force), power-of-two scaling is exact;
  * an order pin (1 + 2^-24 + 2^-24 depends on the order of the adds);
  * IEEE signed-zero rules, +0 pads;
  * Higham's bound on the rank-order sum against exact fp64 sums.
Plus agreement of the two independent oracles (pack-then-loop in C, direct
index in numpy).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import oracle_np
from synth import configs

from _groups import degenerate, mini_sweep, mini_wan, random_group

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x) -> np.ndarray:
    """Exact float -> bf16 bits for values that are representable (asserted)."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not representable in bf16"
    return (u >> 16).astype(np.uint16)


def f32_of(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def grads_from(fn, group):
    """grads[k][i] = bf16 bits of fn(k, i, numel)."""
    return [[bf16_bits(fn(k, i, group.numel(i))) for i in range(group.n_params)]
            for k in range(group.world)]


def valid_mask(group) -> np.ndarray:
    """True where a rank-major position holds data (derived with torch.chunk, not the oracle)."""
    ones = [torch.ones(s, dtype=torch.int16) for s in group.shapes]
    return torch_rank_major(group.world, group.shapes, ones, fill=0).numpy().astype(bool)


def torch_rank_major(world, shapes, tensors, fill):
    """FSDP2-style flat rank-major buffer built from library calls only.

    Each tensor is split along dim 0 with torch.chunk (chunk size ceil(d0/W),
    possibly fewer than W chunks), each rank's chunk is padded to the first
    chunk's row count with `fill`, and ranks are concatenated in order.
    """
    per_rank = [[] for _ in range(world)]
    for shp, t in zip(shapes, tensors):
        t = t.reshape(shp)
        chunks = list(torch.chunk(t, world, dim=0)) if shp[0] > 0 else []
        rows = chunks[0].shape[0] if chunks else 0
        for r in range(world):
            padded = torch.full((rows,) + tuple(shp[1:]), fill, dtype=t.dtype)
            if r < len(chunks):
                padded[: chunks[r].shape[0]] = chunks[r]
            per_rank[r].append(padded.reshape(-1))
    flat = [torch.cat(p) if p else torch.zeros(0, dtype=tensors[0].dtype) for p in per_rank]
    return torch.cat(flat)


def as_i16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())


def groups_for_agreement():
    rng = np.random.default_rng(1234)
    out = [configs.tiny(), degenerate(), mini_wan(), mini_sweep(2), mini_sweep(64),
           configs.qwen3moe(4)]
    for w in (1, 2, 3, 5, 8, 16, 64):
        out.append(random_group(rng, w, int(rng.integers(1, 7))))
    return out


# --------------------------------------------------------------------------- layout


def test_layout_matches_hand_derived_sizes():
    gold = json.load(open(os.path.join(GOLDEN, "layouts.json")))
    for name, g in gold.items():
        if name.startswith("_"):
            continue
        grp = configs.by_name(name)
        assert grp.world == g["W"] and grp.n_params == g["P"]
        L = oracle.layout(grp.world, grp.shapes)
        assert grp.world * grp.n_params == g["chunks"]
        assert sum(grp.numel(i) for i in range(grp.n_params)) == g["N"]
        assert L.Ns == g["Ns"], name
        for key in ("S", "c", "off"):
            if key in g:
                assert getattr(L, key) == g[key]
        if "chunks_under_16KiB" in g:
            assert sum(grp.world for c in L.c if 2 * c < 16384) == g["chunks_under_16KiB"]
            pads = sum(1 for i in range(grp.n_params) for r in range(grp.world)
                       if r * L.c[i] >= grp.numel(i))
            assert pads == g["all_pad_chunks"]
        S, c, off, Ns = oracle_np.layout(grp.world, grp.shapes)
        assert (S, c, off, Ns) == (L.S, L.c, L.off, L.Ns)


def test_worked_example():
    gold = json.load(open(os.path.join(GOLDEN, "worked_w2.json")))
    W, shapes = gold["world"], [tuple(s) for s in gold["shapes"]]
    ag = bf16_bits(np.array(gold["ag_values"], dtype=np.float32))
    params = oracle.ag_copyout(W, shapes, ag)
    for p, exp in zip(params, gold["expected_params"]):
        assert np.array_equal(f32_of(p), np.array(exp, dtype=np.float32))
    grads = [[bf16_bits(np.array(g, dtype=np.float32)) for g in rk] for rk in gold["grads"]]
    for mode, key in ((0, "expected_rs_unscaled"), (1, "expected_rs_scaled")):
        out = oracle.rs_reduce(W, shapes, grads, mode)
        assert np.array_equal(out, np.array(gold[key], dtype=np.float32))
        assert np.array_equal(oracle_np.rs_direct(W, shapes, grads, mode), out)


# --------------------------------------------------------------------------- all-gather


@pytest.mark.parametrize("grp", groups_for_agreement(), ids=lambda g: f"{g.name}_w{g.world}")
def test_ag_copyout_matches_torch_chunk(grp):
    rng = np.random.default_rng(7)
    full = [rng.integers(1, 0x7F00, size=grp.numel(i), dtype=np.uint16) for i in range(grp.n_params)]
    # rank-major buffer with every pad position poisoned (0xFFFF is a bf16 NaN)
    ag = torch_rank_major(grp.world, grp.shapes, [as_i16(x) for x in full], fill=-1)
    ag = ag.numpy().view(np.uint16)
    placed = oracle.ag_copyout(grp.world, grp.shapes, ag)
    L = oracle.layout(grp.world, grp.shapes)
    for i in range(grp.n_params):
        n = grp.numel(i)
        assert placed[i].size == grp.world * L.c[i]
        assert np.array_equal(placed[i][:n], full[i])
        assert np.all(placed[i][n:] == 0)
    direct = oracle_np.ag_direct(grp.world, grp.shapes, ag)
    for a, b in zip(placed, direct):
        assert np.array_equal(a, b)


def test_ag_round_trip():
    grp = configs.tiny()
    L = oracle.layout(grp.world, grp.shapes)
    ag = synth.ag_host(grp, L.Ns, seed=3).reshape(-1)
    mask = valid_mask(grp)
    placed = oracle.ag_copyout(grp.world, grp.shapes, ag)
    # pack the placed params back (slot staging is a bf16 pack): equals ag on valid positions
    back = np.full_like(ag, 0x1234)
    oracle.slot_stage(grp.world, grp.shapes, [p[:grp.numel(i)] for i, p in enumerate(placed)], back)
    assert np.array_equal(back[mask], ag[mask])
    assert np.all(back[~mask] == 0x1234)


# --------------------------------------------------------------------------- gradient pack


@pytest.mark.parametrize("grp", groups_for_agreement(), ids=lambda g: f"{g.name}_w{g.world}")
def test_pack_matches_torch_chunk(grp):
    g = synth.grads_host(grp, seed=5)[0]
    as_f32 = [as_i16(x).view(torch.bfloat16).float() for x in g]   # torch's own bf16 -> fp32
    ref = torch_rank_major(grp.world, grp.shapes, as_f32, fill=0.0).numpy()
    got = oracle.pack_f32(grp.world, grp.shapes, g)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    slot = np.full(ref.size, 0x7777, dtype=np.uint16)
    oracle.slot_stage(grp.world, grp.shapes, g, slot)
    ref16 = torch_rank_major(grp.world, grp.shapes, [as_i16(x) for x in g], fill=0x7777)
    assert np.array_equal(slot, ref16.numpy().view(np.uint16))


# --------------------------------------------------------------------------- reduce-scatter


@pytest.mark.parametrize("grp", groups_for_agreement(), ids=lambda g: f"{g.name}_w{g.world}")
@pytest.mark.parametrize("scale", [0, 1])
def test_two_oracles_agree(grp, scale):
    grads = synth.grads_host(grp, seed=11)
    a = oracle.rs_reduce(grp.world, grp.shapes, grads, scale)
    b = oracle_np.rs_direct(grp.world, grp.shapes, grads, scale)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("seed", range(1, 17))
def test_two_oracles_agree_tiny_seeds(seed):
    grp = configs.tiny()
    grads = synth.grads_host(grp, seed=seed)
    a = oracle.rs_reduce(grp.world, grp.shapes, grads, 1)
    b = oracle_np.rs_direct(grp.world, grp.shapes, grads, 1)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


@pytest.mark.parametrize("W", [1, 2, 3, 4, 8, 16, 64])
def test_identical_ranks_give_W_times_g(W):
    grp = configs.Group("ident", W, ((37, 16), (1000,), (7, 3), (5, 130)))
    g = synth.grads_host(configs.Group("src", 1, grp.shapes), seed=2)[0]
    grads = [g for _ in range(W)]
    out = oracle.rs_reduce(W, grp.shapes, grads, 0)
    scaled = oracle.rs_reduce(W, grp.shapes, grads, 1)
    ref = torch_rank_major(W, grp.shapes, [as_i16(x).view(torch.bfloat16).float() for x in g], 0.0)
    ref = ref.numpy().astype(np.float64)
    assert np.array_equal(out.astype(np.float64), W * ref)          # k*g is exact for k <= 64
    if W & (W - 1) == 0:
        assert np.array_equal(scaled.astype(np.float64), ref)       # 1/W is a power of two


@pytest.mark.parametrize("W,hot", [(4, 0), (4, 3), (8, 5), (16, 15)])
def test_one_hot_rank(W, hot):
    grp = configs.Group("onehot", W, ((37, 16), (1000,), (256, 3)))
    g = synth.grads_host(configs.Group("src", 1, grp.shapes), seed=9)[0]
    zero = [np.zeros_like(x) for x in g]
    grads = [g if k == hot else zero for k in range(W)]
    out = oracle.rs_reduce(W, grp.shapes, grads, 0)
    ref = torch_rank_major(W, grp.shapes, [as_i16(x).view(torch.bfloat16).float() for x in g], 0.0)
    assert np.array_equal(out, ref.numpy())


@pytest.mark.parametrize("W", [2, 3, 8, 64])
def test_small_integers_sum_exactly(W):
    grp = configs.Group("ints", W, ((65, 9), (301,), (3, 3)))
    rng = np.random.default_rng(W)
    ints = [[rng.integers(-8, 9, size=grp.numel(i)) for i in range(grp.n_params)] for _ in range(W)]
    grads = [[bf16_bits(m.astype(np.float32) * np.float32(2.0 ** -10)) for m in rk] for rk in ints]
    out = oracle.rs_reduce(W, grp.shapes, grads, 0)
    # brute force in int64, laid out by the torch.chunk builder
    tot = [sum(ints[k][i] for k in range(W)).astype(np.int64) for i in range(grp.n_params)]
    ref = torch_rank_major(W, grp.shapes, [torch.from_numpy(t) for t in tot], 0).numpy()
    assert np.array_equal(out.astype(np.float64), ref.astype(np.float64) * 2.0 ** -10)


def test_rank_order_is_fixed():
    # fp32: (1 + 2^-24) + 2^-24 == 1, but 1 + (2^-24 + 2^-24) == 1 + 2^-23.
    shapes = ((3,),)
    tiny_v, one = 2.0 ** -24, 1.0
    def run(vals):
        grads = [[bf16_bits(np.full(3, v, dtype=np.float32))] for v in vals]
        return oracle.rs_reduce(3, shapes, grads, 0)[0], oracle_np.rs_direct(3, shapes, grads, 0)[0]
    assert run([one, tiny_v, tiny_v]) == (np.float32(1.0), np.float32(1.0))
    assert run([tiny_v, tiny_v, one]) == (np.float32(1.0 + 2.0 ** -23),) * 2
    vals = [bf16_bits(np.float32(v)) for v in (one, tiny_v, tiny_v)]
    assert oracle.sum_ranks(np.array(vals), 0) == np.float32(1.0)


def test_signed_zero_and_pads():
    W = 4
    shapes = ((5, 2), (3,))          # rank 3 of the first param and ranks 3.. of the second pad
    neg = [[np.full(10, 0x8000, np.uint16), np.full(3, 0x8000, np.uint16)] for _ in range(W)]
    out = oracle.rs_reduce(W, shapes, neg, 0).view(np.uint32)
    mask = valid_mask(configs.Group("z", W, shapes))
    assert np.all(out[mask] == 0x80000000)          # -0 + -0 = -0 (sum starts from g_0)
    assert np.all(out[~mask] == 0)                  # pads are +0
    mixed = [neg[0]] + [[np.zeros(10, np.uint16), np.zeros(3, np.uint16)] for _ in range(W - 1)]
    out = oracle.rs_reduce(W, shapes, mixed, 0).view(np.uint32)
    assert np.all(out == 0)                         # -0 + +0 = +0


@pytest.mark.parametrize("W", [2, 4, 8, 16, 32, 64])
def test_power_of_two_scale_is_exact(W):
    grp = configs.Group("scale", W, ((3 * W + 1, 5), (2 * W,)))
    grads = synth.grads_host(grp, seed=4)
    a = oracle.rs_reduce(W, grp.shapes, grads, 0).astype(np.float64)
    b = oracle.rs_reduce(W, grp.shapes, grads, 1).astype(np.float64)
    assert np.array_equal(b, a / W)


@pytest.mark.parametrize("grp", [configs.tiny(), mini_wan(), mini_sweep(64)], ids=lambda g: g.name)
def test_higham_bound_and_tree_tolerance(grp):
    W = grp.world
    grads = synth.grads_host(grp, seed=21)
    E, A = oracle.exact_f64(W, grp.shapes, grads)
    out = oracle.rs_reduce(W, grp.shapes, grads, 0).astype(np.float64)
    u = 2.0 ** -24
    assert np.all(np.abs(out - E) <= (W - 1) * u * A)
    # a pairwise (tree) order stays inside ceil(log2 W) * u * A, hence inside 1e-6 * A
    L = oracle.layout(W, grp.shapes)
    tree = np.zeros(W * L.Ns, dtype=np.float64)
    for i in range(grp.n_params):
        for r in range(W):
            lo, hi = r * L.c[i], min((r + 1) * L.c[i], grp.numel(i))
            if hi > lo:
                terms = [f32_of(grads[k][i][lo:hi]) for k in range(W)]
                s = r * L.Ns + L.off[i]
                tree[s: s + hi - lo] = oracle_np.tree_sum(terms)
    bound = max(1, math.ceil(math.log2(W))) * u * A
    assert np.all(np.abs(tree - E) <= bound)
    assert np.all(bound <= 1e-6 * A)


def test_gloo_reduce_scatter_agrees(tmp_path):
    """torch.distributed.reduce_scatter_tensor (gloo, 4 processes) on FSDP2-packed fp32 buffers."""
    from _dist_helpers import run_gloo_reduce_scatter
    grp = configs.tiny()
    W = grp.world
    rng = np.random.default_rng(3)
    ints = [[rng.integers(-8, 9, size=grp.numel(i)) for i in range(grp.n_params)] for _ in range(W)]
    exact = [[bf16_bits(m.astype(np.float32) * np.float32(2.0 ** -10)) for m in rk] for rk in ints]
    general = synth.grads_host(grp, seed=8)
    for grads, bitwise in ((exact, True), (general, False)):
        packed = [torch_rank_major(W, grp.shapes,
                                   [as_i16(x).view(torch.bfloat16).float() for x in grads[k]], 0.0)
                  for k in range(W)]
        shards = run_gloo_reduce_scatter([p.numpy() for p in packed], tmp_path)
        got = np.concatenate(shards)
        out = oracle.rs_reduce(W, grp.shapes, grads, 0)
        if bitwise:
            assert np.array_equal(got.view(np.uint32), out.view(np.uint32))
        else:
            E, A = oracle.exact_f64(W, grp.shapes, grads)
            u = 2.0 ** -24
            assert np.all(np.abs(got - E) <= (W - 1) * u * A)
            assert np.all(np.abs(out - E) <= (W - 1) * u * A)


# --------------------------------------------------------------------------- slot-reuse


@pytest.mark.parametrize("grp", [configs.tiny(), mini_wan(), degenerate()], ids=lambda g: g.name)
def test_slot_reuse_equals_plain(grp):
    W = grp.world
    L = oracle.layout(W, grp.shapes)
    grads = synth.grads_host(grp, seed=13)
    slots = [np.full(W * L.Ns, 0xFFFF, dtype=np.uint16) for _ in range(W)]  # stale AG data: NaN
    for k in range(W):
        oracle.slot_stage(W, grp.shapes, grads[k], slots[k])
    for scale in (0, 1):
        a = oracle.rs_reduce_slots(W, grp.shapes, slots, scale)
        b = oracle.rs_reduce(W, grp.shapes, grads, scale)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


# --------------------------------------------------------------------------- per-element helpers


@pytest.mark.parametrize("grp", [configs.tiny(), degenerate(), mini_wan()], ids=lambda g: g.name)
def test_locate_and_ag_source_agree_with_bulk(grp):
    W = grp.world
    L = oracle.layout(W, grp.shapes)
    grads = synth.grads_host(grp, seed=17)
    out = oracle.rs_reduce(W, grp.shapes, grads, 1)
    rng = np.random.default_rng(0)
    for flat in rng.integers(0, max(1, W * L.Ns), size=min(400, W * L.Ns)):
        r, j = divmod(int(flat), L.Ns)
        st, i, src = oracle.locate(W, grp.shapes, r, j)
        if st == 1:
            v = oracle.sum_ranks(np.array([grads[k][i][src] for k in range(W)]), 1)
            assert v.view(np.uint32) == out[flat].view(np.uint32)
        else:
            assert st == 0 and out[flat].view(np.uint32) == 0
    ag = synth.ag_host(grp, L.Ns, seed=2).reshape(-1)
    placed = oracle.ag_copyout(W, grp.shapes, ag)
    for i in range(grp.n_params):
        for q in rng.integers(0, max(1, W * L.c[i]), size=min(50, W * L.c[i])):
            st, a = oracle.ag_source(W, grp.shapes, i, int(q))
            assert placed[i][q] == (ag[a] if st == 1 else 0)


# --------------------------------------------------------------------------- tree order
# The tree order is an optional mode of the reduction: adjacent pairs level by level, an
# odd last value carried.  Pinned by worked values where it differs from the rank order,
# by a top-down formulation of the same tree, by closed forms and by its error bound.

E24 = 2.0 ** -24


def _tree_bits(vals):
    return [int(bf16_bits(np.float32(v))) for v in vals]


@pytest.mark.parametrize("vals,tree,rank", [
    ([1.0, E24, E24, E24], 1.0 + 2.0 ** -23, 1.0),        # (1+e) + (e+e): the pair of e's survives
    ([E24, E24, 1.0], 1.0 + 2.0 ** -23, 1.0 + 2.0 ** -23),
    ([1.0, E24, E24], 1.0, 1.0),                           # (1+e) rounds to 1, then + e rounds to 1
    # [1, 2e, e] -> [1+2^-23, e] -> 1 + 3e, a tie, rounds to the even 1 + 2^-22
    ([1.0, E24, E24, E24, E24], 1.0 + 2.0 ** -22, 1.0),
    ([-0.0, -0.0, -0.0], -0.0, -0.0),
])
def test_tree_worked_values(vals, tree, rank):
    bits = np.array(_tree_bits(vals), dtype=np.uint16)
    got = oracle.sum_ranks_tree(bits, 0)
    assert got.view(np.uint32) == np.float32(tree).view(np.uint32)
    assert oracle.sum_ranks(bits, 0).view(np.uint32) == np.float32(rank).view(np.uint32)


def _top_down(v):
    """The same tree written top-down: split at the largest power of two below n."""
    n = len(v)
    if n == 1:
        return v[0]
    p = 1
    while 2 * p < n:
        p *= 2
    return np.float32(_top_down(v[:p]) + _top_down(v[p:]))


@pytest.mark.parametrize("W", list(range(1, 34)) + [63, 64, 65, 100])
def test_tree_matches_top_down_split(W):
    rng = np.random.default_rng(W)
    for _ in range(40):
        # wide exponent range and mixed signs, so that the grouping changes the rounding
        mant = rng.integers(128, 256, size=W).astype(np.float32) / np.float32(128.0)
        exps = rng.integers(-30, 2, size=W)
        sign = np.where(rng.random(W) < 0.3, -1.0, 1.0).astype(np.float32)
        f = (sign * mant * np.float32(2.0) ** exps).astype(np.float32)
        bits = bf16_bits(f)
        want = _top_down([np.float32(x) for x in f32_of(bits)])
        assert oracle.sum_ranks_tree(bits, 0).view(np.uint32) == np.float32(want).view(np.uint32)
        scaled = np.float32(np.float32(want) * np.float32(1.0 / W))
        assert oracle.sum_ranks_tree(bits, 1).view(np.uint32) == scaled.view(np.uint32)


@pytest.mark.parametrize("grp", groups_for_agreement(), ids=lambda g: f"{g.name}_w{g.world}")
def test_tree_reduce_matches_numpy_levels(grp):
    """The C tree reduce-scatter against the numpy levels tree, chunk by chunk (pads +0)."""
    W = grp.world
    grads = synth.grads_host(grp, seed=23)
    out = oracle.rs_reduce_tree(W, grp.shapes, grads, 1)
    L = oracle.layout(W, grp.shapes)
    ref = np.zeros(W * L.Ns, dtype=np.float32)
    for i in range(grp.n_params):
        for r in range(W):
            lo, hi = r * L.c[i], min((r + 1) * L.c[i], grp.numel(i))
            if hi > lo:
                s = r * L.Ns + L.off[i]
                tree = oracle_np.tree_sum([f32_of(grads[k][i][lo:hi]) for k in range(W)])
                ref[s: s + hi - lo] = tree * np.float32(1.0 / W)
    assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("W", [1, 2, 3, 8, 16, 64])
def test_tree_closed_forms_and_bound(W):
    grp = configs.Group("treecf", W, ((37, 16), (1000,), (7, 3)))
    g = synth.grads_host(configs.Group("src", 1, grp.shapes), seed=2)[0]
    same = oracle.rs_reduce_tree(W, grp.shapes, [g for _ in range(W)], 0).astype(np.float64)
    plain = oracle.rs_reduce(W, grp.shapes, [g for _ in range(W)], 0).astype(np.float64)
    assert np.array_equal(same, plain)             # k*g is exact for k <= 64: any order agrees
    grads = synth.grads_host(grp, seed=22)
    E, A = oracle.exact_f64(W, grp.shapes, grads)
    tree = oracle.rs_reduce_tree(W, grp.shapes, grads, 0).astype(np.float64)
    assert np.all(np.abs(tree - E) <= max(1, math.ceil(math.log2(W))) * E24 * A)


@pytest.mark.parametrize("W", [2, 3, 8, 64])
def test_exact_sums_against_integer_brute_force(W):
    """The exact fp64 sums behind every tolerance check: small integers times 2^-10, summed
    in int64 and laid out with torch.chunk, give E and A exactly; pads give 0."""
    grp = configs.Group("exact", W, ((65, 9), (301,), (3, 3)))
    rng = np.random.default_rng(100 + W)
    ints = [[rng.integers(-8, 9, size=grp.numel(i)) for i in range(grp.n_params)] for _ in range(W)]
    grads = [[bf16_bits(m.astype(np.float32) * np.float32(2.0 ** -10)) for m in rk] for rk in ints]
    E, A = oracle.exact_f64(W, grp.shapes, grads)
    tot = [sum(ints[k][i] for k in range(W)).astype(np.int64) for i in range(grp.n_params)]
    mag = [sum(np.abs(ints[k][i]) for k in range(W)).astype(np.int64) for i in range(grp.n_params)]
    e_ref = torch_rank_major(W, grp.shapes, [torch.from_numpy(t) for t in tot], 0).numpy()
    a_ref = torch_rank_major(W, grp.shapes, [torch.from_numpy(t) for t in mag], 0).numpy()
    assert np.array_equal(E, e_ref.astype(np.float64) * 2.0 ** -10)
    assert np.array_equal(A, a_ref.astype(np.float64) * 2.0 ** -10)


# --------------------------------------------------------------------------- fp32 gradients


def _f32_grads_of(grads):
    """The fp32 values of bf16 gradients (the widening is exact)."""
    return [[f32_of(g) for g in rk] for rk in grads]


@pytest.mark.parametrize("grp", [configs.tiny(), mini_wan(), degenerate(), mini_sweep(64)]
                         + [random_group(np.random.default_rng(77 + w), w, 4) for w in (1, 3, 5, 16)],
                         ids=lambda g: f"{g.name}_w{g.world}")
def test_f32_inputs_holding_bf16_values_give_the_bf16_results(grp):
    """fp32 gradients whose values are bf16 values reduce to the pinned bf16 results, bit for
    bit, directly and through fp32 slots (stale slot contents: NaN)."""
    W = grp.world
    L = oracle.layout(W, grp.shapes)
    grads = synth.grads_host(grp, seed=31)
    g32 = _f32_grads_of(grads)
    slots = [np.full(W * L.Ns, 0xFFFFFFFF, dtype=np.uint32) for _ in range(W)]
    for k in range(W):
        oracle.slot_stage_f32(W, grp.shapes, g32[k], slots[k])
    for scale in (0, 1):
        want = oracle.rs_reduce(W, grp.shapes, grads, scale).view(np.uint32)
        assert np.array_equal(oracle.rs_reduce_f32(W, grp.shapes, g32, scale).view(np.uint32), want)
        assert np.array_equal(oracle.rs_reduce_slots_f32(W, grp.shapes, slots, scale).view(np.uint32),
                              want)


@pytest.mark.parametrize("W", [1, 2, 3, 8, 64])
def test_f32_sums_keep_bits_below_bf16_precision(W):
    """Multiples of 2^-20 around 1 (not bf16 values) sum exactly: int64 brute force, laid out
    by the torch.chunk builder.  A pack or a staging that drops the low 16 bits fails."""
    grp = configs.Group("f32ints", W, ((65, 9), (301,), (3, 3)))
    rng = np.random.default_rng(100 + W)
    ints = [[rng.integers(-8, 9, size=grp.numel(i)) + (2 ** 20 if k == 0 else 0)
             for i in range(grp.n_params)] for k in range(W)]
    g32 = [[(m.astype(np.float64) * 2.0 ** -20).astype(np.float32) for m in rk] for rk in ints]
    assert np.array_equal(g32[0][0].astype(np.float64) * 2 ** 20, ints[0][0])   # exact inputs
    tot = [sum(ints[k][i] for k in range(W)).astype(np.int64) for i in range(grp.n_params)]
    ref = torch_rank_major(W, grp.shapes, [torch.from_numpy(t) for t in tot], 0).numpy()
    ref = ref.astype(np.float64) * 2.0 ** -20
    assert np.array_equal(oracle.rs_reduce_f32(W, grp.shapes, g32, 0).astype(np.float64), ref)
    L = oracle.layout(W, grp.shapes)
    slots = [np.zeros(W * L.Ns, dtype=np.float32) for _ in range(W)]
    for k in range(W):
        oracle.slot_stage_f32(W, grp.shapes, g32[k], slots[k])
    assert np.array_equal(oracle.rs_reduce_slots_f32(W, grp.shapes, slots, 0).astype(np.float64), ref)


def test_f32_rank_order_is_fixed_and_signed_zeros():
    shapes = ((3,),)
    def run(vals):
        return oracle.rs_reduce_f32(3, shapes, [[np.full(3, v, dtype=np.float32)] for v in vals], 0)[0]
    assert run([1.0, 2.0 ** -24, 2.0 ** -24]) == np.float32(1.0)
    assert run([2.0 ** -24, 2.0 ** -24, 1.0]) == np.float32(1.0 + 2.0 ** -23)
    W, shapes = 4, ((5, 2), (3,))
    neg = [[np.full(10, -0.0, np.float32), np.full(3, -0.0, np.float32)] for _ in range(W)]
    out = oracle.rs_reduce_f32(W, shapes, neg, 0).view(np.uint32)
    mask = valid_mask(configs.Group("z", W, shapes))
    assert np.all(out[mask] == 0x80000000) and np.all(out[~mask] == 0)


@pytest.mark.parametrize("grp", [configs.tiny(), degenerate()], ids=lambda g: g.name)
def test_f32_slot_stage_matches_torch_chunk(grp):
    """Staging one rank's fp32 gradients: the torch.chunk builder's rank-major buffer at valid
    positions, the slot's old words (NaN) at pads."""
    W = grp.world
    L = oracle.layout(W, grp.shapes)
    rng = np.random.default_rng(5)
    g = [rng.standard_normal(grp.numel(i)).astype(np.float32) for i in range(grp.n_params)]
    slot = np.full(W * L.Ns, 0xFFFFFFFF, dtype=np.uint32)
    oracle.slot_stage_f32(W, grp.shapes, g, slot)
    ref = torch_rank_major(W, grp.shapes, [torch.from_numpy(x.view(np.int32)) for x in g], -1).numpy()
    mask = valid_mask(grp)
    assert np.array_equal(slot[mask], ref.view(np.uint32)[mask])
    assert np.all(slot[~mask] == 0xFFFFFFFF)


def test_f32_gloo_reduce_scatter_agrees(tmp_path):
    """torch.distributed.reduce_scatter_tensor (gloo, 4 processes) on FSDP2-packed fp32
    buffers of fp32 gradients: bit for bit on exact sums, within the fp32 bound otherwise."""
    from _dist_helpers import run_gloo_reduce_scatter
    grp = configs.tiny()
    W = grp.world
    rng = np.random.default_rng(6)
    exact = [[((rng.integers(-8, 9, size=grp.numel(i)) + 2 ** 20) * 2.0 ** -20).astype(np.float32)
              for i in range(grp.n_params)] for _ in range(W)]
    general = [[rng.standard_normal(grp.numel(i)).astype(np.float32) * np.float32(1e-3)
                for i in range(grp.n_params)] for _ in range(W)]
    for grads, bitwise in ((exact, True), (general, False)):
        packed = [torch_rank_major(W, grp.shapes, [torch.from_numpy(x) for x in grads[k]], 0.0)
                  for k in range(W)]
        got = np.concatenate(run_gloo_reduce_scatter([p.numpy() for p in packed], tmp_path))
        out = oracle.rs_reduce_f32(W, grp.shapes, grads, 0)
        if bitwise:
            assert np.array_equal(got.view(np.uint32), out.view(np.uint32))
        else:
            ex = torch_rank_major(W, grp.shapes, [torch.from_numpy(sum(grads[k][i].astype(np.float64)
                                                                      for k in range(W)))
                                                  for i in range(grp.n_params)], 0.0).numpy()
            mag = torch_rank_major(W, grp.shapes, [torch.from_numpy(sum(np.abs(grads[k][i]).astype(np.float64)
                                                                       for k in range(W)))
                                                   for i in range(grp.n_params)], 0.0).numpy()
            bound = (W - 1) * 2.0 ** -24 * mag
            assert np.all(np.abs(got - ex) <= bound) and np.all(np.abs(out - ex) <= bound)


@pytest.mark.parametrize("grp", groups_for_agreement(), ids=lambda g: f"{g.name}_w{g.world}")
def test_two_oracles_agree_on_f32_gradients(grp):
    """The C oracle's fp32 pack-then-sum and the numpy direct-index definition, bit for bit,
    on random fp32 gradients with a wide exponent range."""
    rng = np.random.default_rng(grp.world * 7 + grp.n_params)
    grads = [[(rng.standard_normal(grp.numel(i)) * np.exp2(rng.integers(-30, 10, size=grp.numel(i))))
              .astype(np.float32) for i in range(grp.n_params)] for _ in range(grp.world)]
    for scale in (0, 1):
        a = oracle.rs_reduce_f32(grp.world, grp.shapes, grads, scale)
        b = oracle_np.rs_direct_f32(grp.world, grp.shapes, grads, scale)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
