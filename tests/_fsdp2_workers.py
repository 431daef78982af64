"""A rank of a real FSDP2 job on the CPU (gloo) whose collectives are wrapped to capture
the buffers FSDP2 itself builds: the all-gather output (the rank-major bf16 buffer) and
the reduce-scatter input and output (the packed fp32 gradients and this rank's shard)."""
import datetime
import os

import numpy as np


def integer_grads(shapes, rank):
    """Per-param gradients of one rank: small integers times 2^-10 (exact in bf16, and
    their sums are exact in fp32 in any order)."""
    rng = np.random.default_rng(1000 + rank)
    return [(rng.integers(-8, 9, size=int(np.prod(s))).astype(np.float32) * np.float32(2.0 ** -10))
            .reshape(s) for s in shapes]


def param_values(shapes):
    """Full parameter values, exact in bf16."""
    rng = np.random.default_rng(7)
    return [(rng.integers(-64, 65, size=int(np.prod(s))).astype(np.float32) * np.float32(2.0 ** -6))
            .reshape(s) for s in shapes]


def fsdp2_worker(rank, world, port, shapes, out_dir, reduce_fp32=True, average=False):
    import torch
    import torch.distributed as dist
    from torch.distributed.device_mesh import init_device_mesh
    from torch.distributed.fsdp import MixedPrecisionPolicy, fully_shard
    from torch.distributed.fsdp._fully_shard._fsdp_collectives import (DefaultAllGather,
                                                                       DefaultReduceScatter)

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        captured = {}

        class CaptureAllGather(DefaultAllGather):
            def __call__(self, output_tensor, input_tensor, group, async_op=False):
                super().__call__(output_tensor, input_tensor, group, async_op=False)
                captured.setdefault("ag", output_tensor.detach().clone())
                return None

        class CaptureReduceScatter(DefaultReduceScatter):
            def __call__(self, output_tensor, input_tensor, group, op, async_op=False):
                captured["rs_in"] = input_tensor.detach().clone()
                super().__call__(output_tensor, input_tensor, group, op, async_op=False)
                captured["rs_out"] = output_tensor.detach().clone()
                return None

        class Group(torch.nn.Module):
            def __init__(self):
                super().__init__()
                self.ps = torch.nn.ParameterList(
                    [torch.nn.Parameter(torch.from_numpy(v)) for v in param_values(shapes)])

            def forward(self, gs):
                return sum((p * g).sum() for p, g in zip(self.ps, gs))

        model = Group()
        mesh = init_device_mesh("cpu", (world,))
        fully_shard(model, mesh=mesh,
                    mp_policy=MixedPrecisionPolicy(
                        param_dtype=torch.bfloat16,
                        reduce_dtype=torch.float32 if reduce_fp32 else torch.bfloat16))
        model.set_custom_all_gather(CaptureAllGather())
        model.set_custom_reduce_scatter(CaptureReduceScatter())
        if not average:
            model.set_gradient_divide_factor(1.0)   # a plain sum
        model.set_force_sum_reduction_for_comms(True)   # gloo: SUM, then FSDP2's own division
        gs = [torch.from_numpy(g).to(torch.bfloat16) for g in integer_grads(shapes, rank)]
        model(gs).backward()
        np.save(os.path.join(out_dir, f"ag_{rank}.npy"),
                captured["ag"].view(torch.int16).numpy().view(np.uint16))
        rs_in = captured["rs_in"]
        if rs_in.dtype == torch.bfloat16:
            np.save(os.path.join(out_dir, f"rs_in_bf16_{rank}.npy"), rs_in.view(torch.int16).numpy().view(np.uint16))
        np.save(os.path.join(out_dir, f"rs_in_{rank}.npy"), rs_in.float().numpy())
        np.save(os.path.join(out_dir, f"rs_out_{rank}.npy"), captured["rs_out"].float().numpy())
        for i, p in enumerate(model.ps):          # the reduced gradient FSDP2 hands to the optimizer
            np.save(os.path.join(out_dir, f"grad_{rank}_{i}.npy"), p.grad.to_local().float().numpy())
    finally:
        dist.destroy_process_group()
