"""Helpers for the GPU parity tests: moving bf16 bit patterns to and from the device."""
import numpy as np
import torch


def to_dev(bits: np.ndarray, shape=None, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(torch.bfloat16)
    if shape is not None:
        t = t.reshape(shape)
    return t.to(device)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().reshape(-1).view(np.uint16)


def f32_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().reshape(-1).view(np.uint32)


def grads_to_dev(group, grads_host):
    return [[to_dev(grads_host[k][i], group.shapes[i]) for i in range(group.n_params)]
            for k in range(group.world)]


def padded_params(plan, group, fill=0x7777, device="cuda"):
    """Fresh padded parameter storage, pre-filled with a marker that is not +0."""
    out = []
    for i in range(group.n_params):
        n = plan.query(i)["padded_numel"]
        t = torch.full((n,), fill, dtype=torch.int16, device=device).view(torch.bfloat16)
        out.append(t)
    return out


def poison_pads(ag_bits: np.ndarray, group, layout) -> np.ndarray:
    """Set every pad position of a rank-major buffer to 0xFFFF (a bf16 NaN)."""
    ag = ag_bits.copy().reshape(group.world, layout.Ns)
    for i in range(group.n_params):
        for r in range(group.world):
            valid = max(0, min(layout.c[i], group.numel(i) - r * layout.c[i]))
            ag[r, layout.off[i] + valid: layout.off[i] + layout.c[i]] = 0xFFFF
    return ag.reshape(-1)
