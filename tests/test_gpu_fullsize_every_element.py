"""GPU parity at full size, every element, in the benchmark's launch configuration: the three
model-shaped groups and every group of the W sweep (W = 2 ... 64, 34 GB of gradients at 64).

TIDE-RS (weekinpapers.com, Abstract: per-parameter bf16 gradients reduced into
fp32 rank-major shards) and TIDE-AG (same Abstract: the all-gather result lands
in per-parameter storage) run once over the whole group on the device, exactly
as the benchmark calls them.  The oracle then runs param by param: a param's
outputs depend on that param's inputs only (its chunk of every shard, its own
padded storage), so a one-param group over the same W gives the same bits at
those positions.  Every valid and pad element of every fp32 shard and of every
padded parameter is compared bit for bit.  Inputs for the oracle are
regenerated on the host by the generator whose device twin filled the device
buffers.
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


CASES = [(n, T.TIDE_ORDER_RANK) for n in ["llama70b", "qwen3moe", "wan14b"] +
         [f"sweep_w{w}" for w in configs.SWEEP_WORLDS]] + \
        [(n, T.TIDE_ORDER_TREE) for n in ["llama70b", "qwen3moe", "wan14b"]]


@pytest.mark.parametrize("name,order", CASES,
                         ids=[f"{n}_{'tree' if o else 'rank'}" for n, o in CASES])
def test_every_element_rs_and_ag(name, order):
    """Rank order against the oracle's reduce-scatter; tree order (the 32-byte tree kernels
    on these groups) against the oracle's tree sums."""
    group = configs.by_name(name)
    rs_oracle = oracle.rs_reduce if order == T.TIDE_ORDER_RANK else oracle.rs_reduce_tree
    W = group.world
    torch.cuda.empty_cache()
    plan = T.Plan(group.shapes, W)
    L = oracle.layout(W, group.shapes)
    assert plan.shard_numel == L.Ns

    grads = synth.dev_grads(group, SEED)
    out = torch.full((W * L.Ns,), float("nan"), device="cuda")
    plan.rs_reduce(grads, out, scale_mode=T.TIDE_SCALE_INV_WORLD, order=order)  # the bench's call
    torch.cuda.synchronize()
    plan.check()
    del grads
    ag = synth.dev_ag(group, L.Ns, SEED)
    params = [torch.full((W * L.c[i],), 0x7777, dtype=torch.int16, device="cuda")
              .view(torch.bfloat16) for i in range(group.n_params)]
    plan.ag_place(ag, params)                                         # the benchmark's call
    torch.cuda.synchronize()
    plan.check()
    del ag
    torch.cuda.empty_cache()

    shards = out.view(W, L.Ns)
    checked_rs = checked_ag = 0
    for i in range(group.n_params):
        c = L.c[i]
        if c == 0:
            continue
        sub = (group.shapes[i],)
        # RS: rows off_i .. off_i + c_i of every rank's shard
        g_host = [[synth.grad_host(group, SEED, k, i)] for k in range(W)]
        want = rs_oracle(W, sub, g_host, 1).view(np.uint32)
        del g_host
        got = shards[:, L.off[i]: L.off[i] + c].contiguous().cpu().numpy().reshape(-1).view(np.uint32)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (f"{name} param {i}: {bad.size} RS mismatches, first at rank "
                               f"{bad[0] // c} element {bad[0] % c}")
        checked_rs += got.size
        del got, want
        # AG: the whole padded storage of param i, pads included
        ag_sub = np.concatenate([synth.fill_bf16(c, SEED, synth.STREAM_AG, r, 0, group.param_sigma,
                                                 idx0=L.off[i]) for r in range(W)])
        want_p = oracle.ag_copyout(W, sub, ag_sub)[0]
        got_p = bits_of(params[i])
        bad = np.nonzero(got_p != want_p)[0]
        assert bad.size == 0, f"{name} param {i}: {bad.size} AG mismatches, first at {bad[0]}"
        checked_ag += got_p.size
    assert checked_rs == W * L.Ns
    assert checked_ag == sum(W * ci for ci in L.c)
    del out, params, shards
    torch.cuda.empty_cache()
