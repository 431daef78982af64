"""The C-ABI library on the host (no GPU): exports, plan tables, argument validation.

Plans are built with TIDE_PLAN_HOST_ONLY, which makes every entry point run its
full argument validation and then refuse to launch (TIDE_ERR_DEVICE); data
pointers are fake addresses that validation never dereferences.
"""
import os
import re

import numpy as np
import pytest

import oracle
from fsdp2_layout_aware_b200 import tide as T
from synth import configs

from _groups import degenerate, mini_sweep, mini_wan, random_group

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^TIDE_API\s+[\w\s\*]+?\b(tide_\w+)\s*\(", text, flags=re.M)
    return names


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 13
    lib = T.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert T.tide_abi_version() == 1


def test_status_strings():
    for code in range(0, -8, -1):
        assert T.tide_status_string(code) not in ("", "unknown status")
    assert T.tide_status_string(-99) == "unknown status"


def host_plan(group):
    return T.Plan(group.shapes, group.world, host_only=True)


@pytest.mark.parametrize("name", ["tiny", "llama70b", "qwen3moe", "wan14b", "sweep_w2", "sweep_w64"])
def test_plan_layout_matches_oracle(name):
    g = configs.by_name(name)
    plan = host_plan(g)
    L = oracle.layout(g.world, g.shapes)
    assert plan.shard_numel == L.Ns
    for i in range(g.n_params):
        q = plan.query(i)
        assert q["shard_rows"] == L.S[i]
        assert q["shard_offset"] == L.off[i]
        assert q["chunk_numel"] == L.c[i]
        assert q["padded_numel"] == g.world * L.c[i]
    assert plan.workspace_bytes == 0          # host-only: no device tables


def check_tiles(group):
    plan = host_plan(group)
    L = oracle.layout(group.world, group.shapes)
    tiles = plan.tiles()
    assert len(tiles) == plan.n_tiles
    W, Ns = group.world, L.Ns
    cover = np.zeros(W * Ns, dtype=np.int32)
    last = (-1, -1, -1)
    for t in tiles:
        i, r = t.param, t.rank
        assert 0 <= i < group.n_params and 0 <= r < W
        assert 0 < t.n_total <= T.TIDE_TILE_ELEMS and 0 <= t.n_valid <= t.n_total
        e0 = t.src_off - r * L.c[i]
        assert e0 % T.TIDE_TILE_ELEMS == 0 and 0 <= e0 < L.c[i]
        assert t.dst_off == r * Ns + L.off[i] + e0
        key = (i, r, e0)                             # chunk order: param, rank, position
        assert key > last
        last = key
        assert t.n_valid == min(t.n_total, max(0, group.numel(i) - t.src_off))
        cover[t.dst_off: t.dst_off + t.n_total] += 1
        # validity agrees with the oracle's per-position locate, at both ends
        for e in {0, t.n_total - 1, t.n_valid - 1, t.n_valid}:
            if 0 <= e < t.n_total:
                st, p, src = oracle.locate(W, group.shapes, r, t.dst_off - r * Ns + e)
                assert p == i and src == t.src_off + e and st == (1 if e < t.n_valid else 0)
    assert np.all(cover == 1)                        # every output position exactly once


@pytest.mark.parametrize("group", [configs.tiny(), degenerate(), mini_wan(), mini_sweep(64),
                                   configs.qwen3moe(4), configs.Group("big_chunk", 3, ((40000, 3),))],
                         ids=lambda g: g.name)
def test_tiles_cover_output_exactly_once(group):
    check_tiles(group)


def test_tiles_random_groups():
    rng = np.random.default_rng(99)
    for w in (1, 2, 3, 7, 16, 64, 256):
        check_tiles(random_group(rng, w, int(rng.integers(1, 9)), max_rows=2000))


def test_full_config_tile_counts():
    for name in ("llama70b", "qwen3moe", "wan14b"):
        g = configs.by_name(name)
        plan = host_plan(g)
        L = oracle.layout(g.world, g.shapes)
        expect = sum(g.world * -(-c // T.TIDE_TILE_ELEMS) for c in L.c)
        assert plan.n_tiles == expect


@pytest.mark.parametrize("world,params,status", [
    (0, [(4, 4)], T.TIDE_ERR_INVALID_ARG),
    (T.TIDE_MAX_WORLD + 1, [(4, 4)], T.TIDE_ERR_INVALID_ARG),
    (4, [(-1, 4)], T.TIDE_ERR_INVALID_ARG),
    (4, [(4, -2)], T.TIDE_ERR_INVALID_ARG),
    (4, [(2 ** 40, 2 ** 40)], T.TIDE_ERR_INVALID_ARG),
])
def test_plan_group_rejects(world, params, status):
    st, h = T.tide_plan_group(params, world, 0, T.TIDE_PLAN_HOST_ONLY)
    assert st == status and h is None


def test_plan_group_rejects_unknown_flag_and_empty_group_ok():
    st, _ = T.tide_plan_group([(4, 4)], 2, 0, 0x80)
    assert st == T.TIDE_ERR_INVALID_ARG
    flags = T.TIDE_PLAN_HOST_ONLY | T.TIDE_PLAN_TMA | T.TIDE_PLAN_TEST_TMA_TIMEOUT
    st, h = T.tide_plan_group([(4, 4)], 2, 0, flags)
    assert st == T.TIDE_OK
    assert T.tide_plan_errors(h, 0) == (T.TIDE_ERR_DEVICE, 0)   # host-only: no error word
    T.tide_plan_destroy(h)
    st, h = T.tide_plan_group([], 4, 0, T.TIDE_PLAN_HOST_ONLY)
    assert st == T.TIDE_OK
    st, info = T.tide_plan_info(h)
    assert info["shard_numel"] == 0 and info["n_tiles"] == 0
    T.tide_plan_destroy(h)
    T.tide_plan_destroy(None)


# --------------------------------------------------------------------------- argument validation

BASE = 0x7F0000000000   # fake, 256-byte aligned device addresses; never dereferenced


class Fake:
    """Non-overlapping fake buffers laid out for one call."""

    def __init__(self):
        self.next = BASE

    def buf(self, nbytes):
        p = self.next
        self.next += ((nbytes + 4095) // 4096 + 1) * 4096
        return p


def fake_args(group):
    W, P = group.world, group.n_params
    L = oracle.layout(W, group.shapes)
    f = Fake()
    grads = [f.buf(2 * group.numel(i)) for _ in range(W) for i in range(P)]
    gnum = [group.numel(i) for _ in range(W) for i in range(P)]
    out = f.buf(4 * W * L.Ns)
    ag = f.buf(2 * W * L.Ns)
    params = [f.buf(2 * W * L.c[i]) for i in range(P)]
    pnum = [W * L.c[i] for i in range(P)]
    slots = [f.buf(2 * W * L.Ns) for _ in range(W)]
    return dict(grads=grads, gnum=gnum, out=out, n_out=W * L.Ns, ag=ag, n_ag=W * L.Ns,
                params=params, pnum=pnum, slots=slots, n_slot=W * L.Ns)


def rs(plan, a, **kw):
    args = dict(a)
    args.update(kw)
    return T.tide_rs_reduce(plan.handle, args["grads"], args["gnum"], args["out"], args["n_out"],
                            args.get("scale", 1), args.get("order", 0), args.get("use_slots"),
                            args["n_slot"], args.get("engine", 0), args.get("max_ctas", 0), 0)


def ag(plan, a, **kw):
    args = dict(a)
    args.update(kw)
    return T.tide_ag_place(plan.handle, args["ag"], args["n_ag"], args["params"], args["pnum"],
                           args.get("engine", 0), args.get("max_ctas", 0), 0)


@pytest.fixture(scope="module")
def tiny_plan():
    return host_plan(configs.tiny())


@pytest.fixture
def args():
    return fake_args(configs.tiny())


def test_valid_arguments_reach_the_device_check(tiny_plan, args):
    assert rs(tiny_plan, args) == T.TIDE_ERR_DEVICE
    assert rs(tiny_plan, args, use_slots=args["slots"]) == T.TIDE_ERR_DEVICE
    assert ag(tiny_plan, args) == T.TIDE_ERR_DEVICE
    assert ag(tiny_plan, args, engine=1) == T.TIDE_ERR_DEVICE
    h = tiny_plan.handle
    assert T.tide_rs_stage(h, args["grads"], args["gnum"], args["slots"], args["n_slot"], 0, 0, 0) \
        == T.TIDE_ERR_DEVICE
    assert T.tide_rs_reduce_slots(h, args["slots"], args["n_slot"], args["out"], args["n_out"], 1, 0,
                                  0, 0) == T.TIDE_ERR_DEVICE
    assert T.tide_plan_check(h, 0) == T.TIDE_ERR_DEVICE
    for n_seg, status in ((1, T.TIDE_ERR_DEVICE), (4, T.TIDE_ERR_DEVICE), (0, T.TIDE_ERR_INVALID_ARG),
                          (5, T.TIDE_ERR_INVALID_ARG)):
        assert T.tide_rs_reduce_pipelined(h, args["grads"], args["gnum"], args["out"], args["n_out"], 1,
                                          0, args["slots"], args["n_slot"], n_seg, 0, 0, 0) == status
    assert T.tide_launch_ctas(h, 0, 0)[0] == T.TIDE_ERR_DEVICE


def test_rs_validation(tiny_plan, args):
    E = T
    g = list(args["grads"])
    assert rs(tiny_plan, args, scale=2) == E.TIDE_ERR_INVALID_ARG
    assert rs(tiny_plan, args, order=5) == E.TIDE_ERR_INVALID_ARG
    assert rs(tiny_plan, args, engine=7) == E.TIDE_ERR_INVALID_ARG
    assert rs(tiny_plan, args, max_ctas=-1) == E.TIDE_ERR_INVALID_ARG
    g0 = list(g); g0[3] = 0
    assert rs(tiny_plan, args, grads=g0) == E.TIDE_ERR_INVALID_ARG           # null grad
    g1 = list(g); g1[2] += 1
    assert rs(tiny_plan, args, grads=g1) == E.TIDE_ERR_ALIGNMENT             # odd bf16 address
    n1 = list(args["gnum"]); n1[4] -= 1
    assert rs(tiny_plan, args, gnum=n1) == E.TIDE_ERR_SIZE                  # undersized grad
    assert rs(tiny_plan, args, out=0) == E.TIDE_ERR_INVALID_ARG
    assert rs(tiny_plan, args, out=args["out"] + 2) == E.TIDE_ERR_ALIGNMENT  # fp32 needs 4 bytes
    assert rs(tiny_plan, args, n_out=args["n_out"] - 1) == E.TIDE_ERR_SIZE
    assert rs(tiny_plan, args, out=g[5]) == E.TIDE_ERR_INVALID_ARG           # out aliases a grad
    s = list(args["slots"]); s[1] = s[0] + 64
    assert rs(tiny_plan, args, use_slots=s) == E.TIDE_ERR_INVALID_ARG       # slots overlap
    s = list(args["slots"]); s[2] = g[0]
    assert rs(tiny_plan, args, use_slots=s) == E.TIDE_ERR_INVALID_ARG       # slot aliases a grad
    assert rs(tiny_plan, args, use_slots=args["slots"], n_slot=args["n_slot"] - 8) == E.TIDE_ERR_SIZE
    # grads may alias each other (read only)
    g2 = list(g); g2[1 * 5 + 0] = g[0]
    assert rs(tiny_plan, args, grads=g2) == E.TIDE_ERR_DEVICE


def test_ag_validation(tiny_plan, args):
    E = T
    assert ag(tiny_plan, args, ag=0) == E.TIDE_ERR_INVALID_ARG
    assert ag(tiny_plan, args, ag=args["ag"] + 1) == E.TIDE_ERR_ALIGNMENT
    assert ag(tiny_plan, args, n_ag=args["n_ag"] - 1) == E.TIDE_ERR_SIZE
    p = list(args["params"]); p[2] = 0
    assert ag(tiny_plan, args, params=p) == E.TIDE_ERR_INVALID_ARG
    n = list(args["pnum"]); n[4] -= 1
    assert ag(tiny_plan, args, pnum=n) == E.TIDE_ERR_SIZE
    p = list(args["params"]); p[1] = args["ag"] + 2
    assert ag(tiny_plan, args, params=p) == E.TIDE_ERR_INVALID_ARG          # param aliases ag
    p = list(args["params"]); p[3] = p[0] + 2
    assert ag(tiny_plan, args, params=p) == E.TIDE_ERR_INVALID_ARG          # params overlap
    assert ag(tiny_plan, args, engine=3) == E.TIDE_ERR_INVALID_ARG


def test_null_allowed_only_for_empty_buffers():
    g = degenerate()
    plan = host_plan(g)
    a = fake_args(g)
    empty = [i for i in range(g.n_params) if g.numel(i) == 0]
    assert empty
    grads = list(a["grads"])
    for k in range(g.world):
        for i in empty:
            grads[k * g.n_params + i] = 0
    assert rs(plan, a, grads=grads) == T.TIDE_ERR_DEVICE


def test_tensor_table_marshals_once_in_rank_major_order():
    import torch
    grads = [[torch.zeros(n, dtype=torch.bfloat16) for n in (5, 7, 3)] for _ in range(2)]
    t = T._table(grads)
    flat = [g for row in grads for g in row]
    assert len(t) == 6 and t.min_numel == 3
    assert [t.ptrs[j] for j in range(6)] == [g.data_ptr() for g in flat]
    assert [t.numels[j] for j in range(6)] == [5, 7, 3, 5, 7, 3]
    assert T._table(t) is t                                  # a table passes through
    slots = [torch.zeros(4, dtype=torch.bfloat16), torch.zeros(9, dtype=torch.bfloat16)]
    s = T._table(slots)
    assert [s.ptrs[j] for j in range(2)] == [x.data_ptr() for x in slots] and s.min_numel == 4
    assert len(T._table([])) == 0 and T._table([]).min_numel == 0
    # the marshalled arrays go straight to the C ABI, which validates them (sizes and
    # overlaps) before it finds that a host-only plan has no device
    st, h = T.tide_plan_group([(5, 1), (7, 1), (3, 1)], 2, 0, T.TIDE_PLAN_HOST_ONLY)
    assert st == T.TIDE_OK
    out = torch.zeros(2 * (3 + 4 + 2), dtype=torch.float32)
    assert T.tide_rs_reduce(h, t.ptrs, t.numels, out.data_ptr(), out.numel(), 1, 0, None, 0, 0, 0,
                            0) == T.TIDE_ERR_DEVICE
    short = T.TensorTable([g[:2] for g in flat])
    assert T.tide_rs_reduce(h, short.ptrs, short.numels, out.data_ptr(), out.numel(), 1, 0, None, 0,
                            0, 0, 0) == T.TIDE_ERR_SIZE
    T.tide_plan_destroy(h)


# --------------------------------------------------------------------------- one-rank plans, gathering


@pytest.mark.parametrize("group", [configs.tiny(), degenerate(), mini_wan(), configs.qwen3moe(4),
                                   mini_sweep(64),
                                   configs.Group("w256", 256, ((300, 3), (255,), (1000, 2)))],
                         ids=lambda g: f"{g.name}_w{g.world}")
def test_rank_plan_tiles_are_that_ranks_tiles_inside_its_shard(group):
    W = group.world
    full = host_plan(group)
    L = oracle.layout(W, group.shapes)
    all_tiles = full.tiles()
    for r in range(W):
        plan = T.Plan(group.shapes, W, host_only=True, rank=r)
        assert plan.rank == r and plan.shard_numel == L.Ns
        mine = [t for t in all_tiles if t.rank == r]
        tiles = plan.tiles()
        assert len(tiles) == len(mine) == plan.n_tiles
        cover = np.zeros(L.Ns, dtype=np.int32)
        for t, u in zip(tiles, mine):
            assert (t.param, t.rank, t.src_off, t.n_valid, t.n_total) == \
                   (u.param, u.rank, u.src_off, u.n_valid, u.n_total)
            assert t.dst_off == u.dst_off - r * L.Ns
            cover[t.dst_off: t.dst_off + t.n_total] += 1
        assert np.all(cover == 1)                    # the rank's shard, each position once


def test_rank_plan_arguments():
    g = configs.tiny()
    params = [(s[0], int(np.prod(s[1:])) if len(s) > 1 else 1) for s in g.shapes]
    for rank in (-1, g.world, 99):
        st, h = T.tide_plan_group_rank(params, g.world, rank, 0, T.TIDE_PLAN_HOST_ONLY)
        assert st == T.TIDE_ERR_INVALID_ARG and h is None
    plan = T.Plan(g.shapes, g.world, host_only=True, rank=2)
    a = fake_args(g)
    L = oracle.layout(g.world, g.shapes)
    # its output is one shard: Ns elements are enough, fewer are not
    assert rs(plan, a, n_out=L.Ns) == T.TIDE_ERR_DEVICE
    assert rs(plan, a, n_out=L.Ns - 1) == T.TIDE_ERR_SIZE
    # calls that need every rank's tiles refuse it
    assert rs(plan, a, use_slots=a["slots"]) == T.TIDE_ERR_INVALID_ARG
    assert ag(plan, a) == T.TIDE_ERR_INVALID_ARG
    assert T.tide_rs_stage(plan.handle, a["grads"], a["gnum"], a["slots"], a["n_slot"], 0, 0,
                           0) == T.TIDE_ERR_INVALID_ARG
    assert T.tide_rs_stage_one(plan.handle, a["grads"][:g.n_params], a["gnum"][:g.n_params],
                               a["slots"][0], a["n_slot"], 0, 0, 0) == T.TIDE_ERR_INVALID_ARG
    # the slot reduction takes it: one shard out, read from rank 2's rows of every slot
    assert T.tide_rs_reduce_slots(plan.handle, a["slots"], a["n_slot"], a["out"], L.Ns, 1, 0,
                                  0, 0) == T.TIDE_ERR_DEVICE
    assert T.tide_rs_reduce_slots(plan.handle, a["slots"], a["n_slot"], a["out"], L.Ns - 1, 1, 0,
                                  0, 0) == T.TIDE_ERR_SIZE
    assert T.tide_rs_reduce_slots(plan.handle, a["slots"], a["n_slot"] - 1, a["out"], L.Ns, 1, 0,
                                  0, 0) == T.TIDE_ERR_SIZE
    # the pipelined Slot-Reuse takes it: one shard out, each slot one source rank's row
    def pipe(out_n=L.Ns, slot_n=L.Ns, segs=1):
        return T.tide_rs_reduce_pipelined(plan.handle, a["grads"], a["gnum"], a["out"], out_n, 1, 0,
                                          a["slots"], slot_n, segs, 0, 0, 0)
    assert pipe() == T.TIDE_ERR_DEVICE
    assert pipe(segs=g.world) == T.TIDE_ERR_DEVICE
    assert pipe(segs=g.world + 1) == T.TIDE_ERR_INVALID_ARG
    assert pipe(out_n=L.Ns - 1) == T.TIDE_ERR_SIZE
    assert pipe(slot_n=L.Ns - 1) == T.TIDE_ERR_SIZE
    assert T.tide_ag_gather_place(plan.handle, a["slots"], L.Ns, a["params"], a["pnum"], 0, 0,
                                  0) == T.TIDE_ERR_INVALID_ARG


def test_stage_one_validation(tiny_plan, args):
    P = configs.tiny().n_params
    grads, gnum, slot, n = args["grads"][P:2 * P], args["gnum"][P:2 * P], args["slots"][1], args["n_slot"]

    def stage(g=grads, gn=gnum, sl=slot, ns=n, engine=0, cap=0):
        return T.tide_rs_stage_one(tiny_plan.handle, g, gn, sl, ns, engine, cap, 0)
    assert stage() == T.TIDE_ERR_DEVICE              # valid: stops at the host-only plan
    assert stage(engine=1) == T.TIDE_ERR_DEVICE
    assert stage(engine=2) == T.TIDE_ERR_INVALID_ARG
    assert stage(cap=-1) == T.TIDE_ERR_INVALID_ARG
    assert stage(g=[0] + grads[1:]) == T.TIDE_ERR_INVALID_ARG
    assert stage(g=grads[:2] + [grads[2] + 1] + grads[3:]) == T.TIDE_ERR_ALIGNMENT
    assert stage(gn=gnum[:4] + [gnum[4] - 1]) == T.TIDE_ERR_SIZE
    assert stage(sl=0) == T.TIDE_ERR_INVALID_ARG
    assert stage(sl=slot + 1) == T.TIDE_ERR_ALIGNMENT
    assert stage(ns=n - 1) == T.TIDE_ERR_SIZE
    assert stage(sl=grads[3]) == T.TIDE_ERR_INVALID_ARG      # the slot overlaps a gradient
    assert stage(g=[grads[0]] * P, gn=[max(gnum)] * P) == T.TIDE_ERR_DEVICE   # grads may alias


def test_gather_place_validation(tiny_plan, args):
    g = configs.tiny()
    W = g.world
    L = oracle.layout(W, g.shapes)
    f = Fake()
    f.next = BASE + (1 << 40)                        # clear of the other fake buffers
    shards = [f.buf(2 * L.Ns) for _ in range(W)]

    def gather(sh=shards, n=L.Ns, params=None, engine=0):
        return T.tide_ag_gather_place(tiny_plan.handle, sh, n, params or args["params"], args["pnum"],
                                      engine, 0, 0)
    assert gather() == T.TIDE_ERR_DEVICE             # valid: stops at the host-only plan
    assert gather(engine=1) == T.TIDE_ERR_DEVICE
    assert gather(n=L.Ns - 1) == T.TIDE_ERR_SIZE
    assert gather(sh=[shards[0] + 1] + shards[1:]) == T.TIDE_ERR_ALIGNMENT
    assert gather(sh=[0] + shards[1:]) == T.TIDE_ERR_INVALID_ARG
    assert gather(engine=7) == T.TIDE_ERR_INVALID_ARG
    # a parameter storage overlapping a shard is refused
    assert gather(params=[shards[1]] + args["params"][1:]) == T.TIDE_ERR_INVALID_ARG
    # shards may overlap one another (they are only read)
    assert gather(sh=[shards[0]] * W) == T.TIDE_ERR_DEVICE


@pytest.mark.parametrize("W", [4, 32])   # 5 written spans (direct check), 33 (sorted check)
def test_overlap_decision_matches_brute_force(W):
    """Gradients (read), the output and the slots (written) at random addresses: the call is
    refused exactly when a written buffer overlaps any other buffer."""
    g = configs.Group("ov", W, ((3 * W, 4), (2 * W + 1,), (5, 8)))
    L = oracle.layout(W, g.shapes)
    P = g.n_params
    plan = T.Plan(g.shapes, W, host_only=True)
    sizes = ([2 * g.numel(i) for _ in range(W) for i in range(P)] + [4 * W * L.Ns] +
             [2 * W * L.Ns] * W)
    writes = [False] * (W * P) + [True] * (1 + W)
    window = 4 * sum(sizes)
    rng = np.random.default_rng(W)
    seen = set()
    for trial in range(300):
        if trial % 2:
            lo = [BASE + 16 * int(rng.integers(0, window // 16)) for _ in sizes]
        else:
            # packed in a random order with random gaps (no overlap), then sometimes one
            # buffer moved to start inside another
            lo, at = [0] * len(sizes), BASE
            for k in rng.permutation(len(sizes)):
                lo[k] = at
                at += (sizes[k] + 15) // 16 * 16 + 16 * int(rng.integers(0, 4))
            if rng.random() < 0.5:
                a, b = rng.choice(len(sizes), size=2, replace=False)
                lo[a] = lo[b] + 16 * int(rng.integers(0, max(1, sizes[b] // 16)))
        bad = any((writes[a] or writes[b]) and lo[a] < lo[b] + sizes[b] and lo[b] < lo[a] + sizes[a]
                  for a in range(len(sizes)) for b in range(a + 1, len(sizes)))
        st = T.tide_rs_reduce(plan.handle, lo[: W * P], [g.numel(i) for _ in range(W) for i in range(P)],
                              lo[W * P], W * L.Ns, 1, 0, lo[W * P + 1:], W * L.Ns, 0, 0, 0)
        assert st == (T.TIDE_ERR_INVALID_ARG if bad else T.TIDE_ERR_DEVICE)
        seen.add(bad)
    assert seen == {True, False}


def test_short_lived_ctas_take_no_cta_cap(args):
    """Under TIDE_PLAN_SHORT_CTAS the grid is one CTA per unit of work: a CTA cap is refused
    before the device check, and without one the call validates as usual."""
    plan = T.Plan(configs.tiny().shapes, 4, host_only=True, short_ctas=True)
    assert rs(plan, args, max_ctas=8) == T.TIDE_ERR_INVALID_ARG
    assert ag(plan, args, max_ctas=8) == T.TIDE_ERR_INVALID_ARG
    assert rs(plan, args) == T.TIDE_ERR_DEVICE
    assert ag(plan, args, engine=1) == T.TIDE_ERR_DEVICE
    h = plan.handle
    assert T.tide_rs_stage(h, args["grads"], args["gnum"], args["slots"], args["n_slot"], 0, 4, 0) \
        == T.TIDE_ERR_INVALID_ARG
    assert T.tide_rs_reduce_slots(h, args["slots"], args["n_slot"], args["out"], args["n_out"], 1, 0,
                                  4, 0) == T.TIDE_ERR_INVALID_ARG
    # unknown flag bits are still refused
    st, _ = T.tide_plan_group([(4, 4)], 4, 0, T.TIDE_PLAN_HOST_ONLY | 64)
    assert st == T.TIDE_ERR_INVALID_ARG


def test_ipc_calls_validate_their_arguments_on_the_host():
    """The peer-mapping calls refuse NULL pointers and negative devices before any CUDA call."""
    st, handle, off, dev = T.tide_ipc_export(0)
    assert st == T.TIDE_ERR_INVALID_ARG and len(handle) == T.TIDE_IPC_HANDLE_BYTES
    assert T.tide_ipc_open(bytes(T.TIDE_IPC_HANDLE_BYTES), -1) == (T.TIDE_ERR_INVALID_ARG, 0)
    assert T.tide_ipc_open(b"short", 0)[0] == T.TIDE_ERR_INVALID_ARG
    assert T.tide_ipc_close(0, 0) == T.TIDE_ERR_INVALID_ARG
    assert T.tide_ipc_close(1 << 40, -1) == T.TIDE_ERR_INVALID_ARG
    assert T.tide_peer_access(3, 3) == (T.TIDE_OK, 1)        # a device always reads itself
    assert T.tide_peer_access(-1, 0)[0] == T.TIDE_ERR_INVALID_ARG


def test_flag_calls_validate_their_arguments_on_the_host():
    f = BASE + 4096
    assert T.tide_flag_signal(0, 1) == T.TIDE_ERR_INVALID_ARG
    assert T.tide_flag_signal(f + 2, 1) == T.TIDE_ERR_ALIGNMENT
    status = BASE + 8192
    assert T.tide_flag_wait([], 1, 1000, status) == T.TIDE_ERR_INVALID_ARG            # n = 0
    assert T.tide_flag_wait([f] * (T.TIDE_MAX_WORLD + 1), 1, 1000, status) == T.TIDE_ERR_INVALID_ARG
    assert T.tide_flag_wait([f], 1, 0, status) == T.TIDE_ERR_INVALID_ARG               # no time limit
    assert T.tide_flag_wait([f], 1, 61 * 10**9, status) == T.TIDE_ERR_INVALID_ARG      # over 60 s
    assert T.tide_flag_wait([f], 1, 1000, 0) == T.TIDE_ERR_INVALID_ARG                 # no status word
    assert T.tide_flag_wait([f], 1, 1000, status + 1) == T.TIDE_ERR_ALIGNMENT
    assert T.tide_flag_wait([f, 0], 1, 1000, status) == T.TIDE_ERR_INVALID_ARG
    assert T.tide_flag_wait([f, f + 6], 1, 1000, status) == T.TIDE_ERR_ALIGNMENT


def f32_args(group):
    """Fake fp32 buffers: one rank's gradients, W fp32 slots, the fp32 output."""
    W, P = group.world, group.n_params
    L = oracle.layout(W, group.shapes)
    f = Fake()
    f.next = BASE + (1 << 41)                        # clear of the other fake buffers
    return dict(grads=[f.buf(4 * group.numel(i)) for i in range(P)],
                gnum=[group.numel(i) for i in range(P)],
                slots=[f.buf(4 * W * L.Ns) for _ in range(W)], n_slot=W * L.Ns,
                out=f.buf(4 * W * L.Ns), n_out=W * L.Ns, Ns=L.Ns)


def test_f32_stage_validation(tiny_plan):
    a = f32_args(configs.tiny())
    g, gn, sl, n = a["grads"], a["gnum"], a["slots"][0], a["n_slot"]

    def stage(g=g, gn=gn, sl=sl, ns=n, cap=0, plan=tiny_plan, engine=0):
        return T.tide_rs_stage_one_f32(plan.handle, g, gn, sl, ns, engine, cap, 0)
    assert stage() == T.TIDE_ERR_DEVICE              # valid: stops at the host-only plan
    assert stage(engine=1) == T.TIDE_ERR_DEVICE
    assert stage(engine=2) == T.TIDE_ERR_INVALID_ARG
    assert stage(cap=-1) == T.TIDE_ERR_INVALID_ARG
    assert stage(g=[0] + g[1:]) == T.TIDE_ERR_INVALID_ARG
    assert stage(g=g[:2] + [g[2] + 2] + g[3:]) == T.TIDE_ERR_ALIGNMENT   # 2-byte aligned is not enough
    assert stage(gn=gn[:4] + [gn[4] - 1]) == T.TIDE_ERR_SIZE
    assert stage(sl=0) == T.TIDE_ERR_INVALID_ARG
    assert stage(sl=sl + 2) == T.TIDE_ERR_ALIGNMENT
    assert stage(ns=n - 1) == T.TIDE_ERR_SIZE
    assert stage(sl=g[3]) == T.TIDE_ERR_INVALID_ARG  # the slot overlaps a gradient
    # a gradient's fp32 bytes end where its bf16 bytes would not: the spans are 4-byte ones
    assert stage(sl=g[4] + 4 * (gn[4] - 1)) == T.TIDE_ERR_INVALID_ARG
    one_rank = T.Plan(configs.tiny().shapes, 4, host_only=True, rank=1)
    assert stage(plan=one_rank) == T.TIDE_ERR_INVALID_ARG


def test_f32_reduce_slots_validation(tiny_plan):
    a = f32_args(configs.tiny())
    sl, n, out, n_out = a["slots"], a["n_slot"], a["out"], a["n_out"]

    def red(sl=sl, ns=n, o=out, no=n_out, scale=1, cap=0, plan=tiny_plan):
        return T.tide_rs_reduce_slots_f32(plan.handle, sl, ns, o, no, scale, cap, 0)
    assert red() == T.TIDE_ERR_DEVICE
    assert red(scale=0) == T.TIDE_ERR_DEVICE
    assert red(scale=2) == T.TIDE_ERR_INVALID_ARG
    assert red(cap=-3) == T.TIDE_ERR_INVALID_ARG
    assert red(sl=None) == T.TIDE_ERR_INVALID_ARG
    assert red(sl=[sl[0] + 2] + sl[1:]) == T.TIDE_ERR_ALIGNMENT
    assert red(sl=sl[:3] + [0]) == T.TIDE_ERR_INVALID_ARG
    assert red(ns=n - 1) == T.TIDE_ERR_SIZE
    assert red(no=n_out - 1) == T.TIDE_ERR_SIZE
    assert red(o=out + 2) == T.TIDE_ERR_ALIGNMENT
    assert red(o=sl[2]) == T.TIDE_ERR_INVALID_ARG     # out overlaps a slot
    assert red(sl=[sl[0]] * 4) == T.TIDE_ERR_DEVICE   # slots may alias (only read)
    # a one-rank plan: one shard out
    one_rank = T.Plan(configs.tiny().shapes, 4, host_only=True, rank=3)
    assert red(plan=one_rank, no=a["Ns"]) == T.TIDE_ERR_DEVICE
    assert red(plan=one_rank, no=a["Ns"] - 1) == T.TIDE_ERR_SIZE


def test_f32_direct_reduce_validation(tiny_plan):
    g = configs.tiny()
    W, P = g.world, g.n_params
    L = oracle.layout(W, g.shapes)
    f = Fake()
    f.next = BASE + (1 << 42)
    grads = [f.buf(4 * g.numel(i)) for _ in range(W) for i in range(P)]
    gnum = [g.numel(i) for _ in range(W) for i in range(P)]
    out = f.buf(4 * W * L.Ns)

    def red(gr=grads, gn=gnum, o=out, no=W * L.Ns, scale=1, cap=0, plan=tiny_plan):
        return T.tide_rs_reduce_f32(plan.handle, gr, gn, o, no, scale, cap, 0)
    assert red() == T.TIDE_ERR_DEVICE
    assert red(scale=0) == T.TIDE_ERR_DEVICE
    assert red(scale=5) == T.TIDE_ERR_INVALID_ARG
    assert red(cap=-1) == T.TIDE_ERR_INVALID_ARG
    assert red(gr=[0] + grads[1:]) == T.TIDE_ERR_INVALID_ARG
    assert red(gr=grads[:7] + [grads[7] + 2] + grads[8:]) == T.TIDE_ERR_ALIGNMENT
    assert red(gn=gnum[:6] + [gnum[6] - 1] + gnum[7:]) == T.TIDE_ERR_SIZE
    assert red(no=W * L.Ns - 1) == T.TIDE_ERR_SIZE
    assert red(o=out + 2) == T.TIDE_ERR_ALIGNMENT
    assert red(o=grads[9]) == T.TIDE_ERR_INVALID_ARG     # out overlaps a gradient
    assert red(gr=[grads[0]] * (W * P), gn=[max(gnum)] * (W * P)) == T.TIDE_ERR_DEVICE  # grads may alias
    one_rank = T.Plan(g.shapes, W, host_only=True, rank=2)
    assert red(plan=one_rank, no=L.Ns) == T.TIDE_ERR_DEVICE
    assert red(plan=one_rank, no=L.Ns - 1) == T.TIDE_ERR_SIZE


def test_f32_bindings_refuse_other_dtypes():
    """The Plan methods of the fp32 calls refuse torch tensors that are not fp32 before any
    call: the C calls count 4-byte elements."""
    import torch
    plan = T.Plan(configs.tiny().shapes, 4, host_only=True)
    g = configs.tiny()
    L = oracle.layout(4, g.shapes)
    bf = [torch.zeros(g.numel(i), dtype=torch.bfloat16) for i in range(g.n_params)]
    f32 = [torch.zeros(g.numel(i)) for i in range(g.n_params)]
    with pytest.raises(TypeError):
        plan.rs_stage_one_f32(bf, torch.zeros(4 * L.Ns))
    with pytest.raises(TypeError):
        plan.rs_stage_one_f32(f32, torch.zeros(4 * L.Ns, dtype=torch.bfloat16))
    with pytest.raises(TypeError):
        plan.rs_reduce_slots_f32([torch.zeros(4 * L.Ns, dtype=torch.bfloat16)] * 4, torch.zeros(4 * L.Ns))
    with pytest.raises(TypeError):
        plan.rs_reduce_slots_f32([torch.zeros(4 * L.Ns)] * 4, torch.zeros(4 * L.Ns, dtype=torch.float16))
    with pytest.raises(TypeError):
        plan.rs_reduce_f32([bf] * 4, torch.zeros(4 * L.Ns))
