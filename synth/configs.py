"""The five synthetic parameter groups the hot path is exercised on.

Shapes only: each group is a world size W and an ordered list of parameter
shapes (dim 0 first).  Nothing here computes a shard, an offset or a sum.

The groups stand in for the models the TIDE pages evaluate on ("The Endgame of
FSDP Communication", weekinpapers.com, Abstract: Llama-3.1 70B, Wan2.2 and
Qwen3-30B-A3B).  No weights or datasets are used; values come from the seeded
generator in this package.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Group:
    name: str
    world: int
    shapes: tuple            # tuple of shape tuples, dim 0 first
    names: tuple = ()        # parameter names, same order
    zero_expert_params: tuple = ()   # per expert e: the param indices zeroed when unrouted
    n_experts: int = 0
    n_zero_experts: int = 0  # per rank
    grad_sigma: float = 1e-3
    param_sigma: float = 0.02

    @property
    def n_params(self) -> int:
        return len(self.shapes)

    def numel(self, i: int) -> int:
        n = 1
        for d in self.shapes[i]:
            n *= d
        return n

    def dim0(self, i: int) -> int:
        return self.shapes[i][0]

    def inner(self, i: int) -> int:
        n = 1
        for d in self.shapes[i][1:]:
            n *= d
        return n


def tiny() -> Group:
    """Five small params over W=4; several shard boundaries break 16-byte alignment."""
    shapes = ((37, 16), (128, 64), (1000,), (7, 3), (256, 256))
    return Group("tiny", 4, shapes, ("p0_37x16", "p1_128x64", "p2_1000", "p3_7x3", "p4_256x256"))


def llama70b() -> Group:
    """One Llama-3.1-70B decoder layer, W=8 (~856M params)."""
    h, kv, ffn = 8192, 1024, 28672
    items = [("q_proj", (h, h)), ("k_proj", (kv, h)), ("v_proj", (kv, h)), ("o_proj", (h, h)),
             ("gate_proj", (ffn, h)), ("up_proj", (ffn, h)), ("down_proj", (h, ffn)),
             ("input_layernorm", (h,)), ("post_attention_layernorm", (h,))]
    return Group("llama70b", 8, tuple(s for _, s in items), tuple(n for n, _ in items))


def qwen3moe(n_experts: int = 128) -> Group:
    """One Qwen3-30B-A3B MoE layer, W=8: 393 params, 3144 chunks; 5% of experts unrouted."""
    h, hq, hkv, inter = 2048, 4096, 512, 768
    items = [("q_proj", (hq, h)), ("k_proj", (hkv, h)), ("v_proj", (hkv, h)), ("o_proj", (h, hq)),
             ("q_norm", (128,)), ("k_norm", (128,)), ("router", (128, h))]
    expert_params = []
    for e in range(n_experts):
        base = len(items)
        items += [(f"experts.{e}.gate_proj", (inter, h)), (f"experts.{e}.up_proj", (inter, h)),
                  (f"experts.{e}.down_proj", (h, inter))]
        expert_params.append((base, base + 1, base + 2))
    items += [("input_layernorm", (h,)), ("post_attention_layernorm", (h,))]
    n_zero = round(0.05 * n_experts)
    return Group("qwen3moe" if n_experts == 128 else f"qwen3moe_e{n_experts}", 8,
                 tuple(s for _, s in items), tuple(n for n, _ in items),
                 zero_expert_params=tuple(expert_params), n_experts=n_experts,
                 n_zero_experts=n_zero)


def wan14b() -> Group:
    """One Wan2.2-style 14B DiT block, W=16: 27 params, modulation 6x5120 leaves ranks 6..15 all pad."""
    d, f = 5120, 13824
    items = []
    for blk in ("self_attn", "cross_attn"):
        for m in ("q", "k", "v", "o"):
            items += [(f"{blk}.{m}.weight", (d, d)), (f"{blk}.{m}.bias", (d,))]
        items += [(f"{blk}.norm_q.weight", (d,)), (f"{blk}.norm_k.weight", (d,))]
    items += [("norm3.weight", (d,)), ("norm3.bias", (d,)),
              ("ffn.0.weight", (f, d)), ("ffn.0.bias", (f,)),
              ("ffn.2.weight", (d, f)), ("ffn.2.bias", (d,)),
              ("modulation", (6, d))]
    return Group("wan14b", 16, tuple(s for _, s in items), tuple(n for n, _ in items))


def sweep(world: int) -> Group:
    """Fixed 4M-element fp32 output shard per rank: 16 params of (64*W) x 4096."""
    shapes = tuple((64 * world, 4096) for _ in range(16))
    return Group(f"sweep_w{world}", world, shapes, tuple(f"p{i}" for i in range(16)))


SWEEP_WORLDS = (2, 4, 8, 16, 32, 64)


def by_name(name: str) -> Group:
    if name.startswith("sweep_w"):
        return sweep(int(name[len("sweep_w"):]))
    if name.startswith("qwen3moe_e"):
        return qwen3moe(int(name[len("qwen3moe_e"):]))
    table = {"tiny": tiny, "llama70b": llama70b, "qwen3moe": qwen3moe, "wan14b": wan14b}
    return table[name]()


ALL = ("tiny", "llama70b", "qwen3moe", "wan14b") + tuple(f"sweep_w{w}" for w in SWEEP_WORLDS)
