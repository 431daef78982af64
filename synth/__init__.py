"""Seeded synthetic inputs (bf16 gradients and all-gather shards).

This module only draws values; it holds none of the sharding, placement or
reduction arithmetic.  The host generator (synth.c) feeds the CPU oracle and
the tests; its device twin (synth_dev.cu) fills multi-GB device buffers with
the same bits for the benchmark and the full-size checks.

Streams: 0 = gradients, 1 = all-gather shards (parameters), 2 = expert routing.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import configs  # noqa: F401  (re-exported)

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libsynth.so")
DEV_LIB = os.path.join(_HERE, "libsynth_dev.so")

STREAM_GRAD = 0
STREAM_AG = 1
STREAM_ROUTING = 2


def build(verbose: bool = False) -> None:
    """Compile the host generator (gcc) and its device twin (nvcc, sm_100a)."""
    host_cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                "-shared", "-o", HOST_LIB, os.path.join(_HERE, "synth.c")]
    dev_cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
               "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-o", DEV_LIB,
               os.path.join(_HERE, "synth_dev.cu")]
    for cmd in (host_cmd, dev_cmd):
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)


_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_LIB):
            build()
        lib = ctypes.CDLL(HOST_LIB)
        u64, i64, f32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_float
        vp = ctypes.c_void_p
        lib.synth_splitmix64.argtypes = [u64]
        lib.synth_splitmix64.restype = u64
        lib.synth_key.argtypes = [u64, u64, u64, u64]
        lib.synth_key.restype = u64
        lib.synth_sigma_scale.argtypes = [ctypes.c_double]
        lib.synth_sigma_scale.restype = f32
        lib.synth_fill_bf16.argtypes = [vp, i64, u64, u64, u64, u64, u64, f32]
        lib.synth_fill_bf16.restype = None
        lib.synth_gather_bf16.argtypes = [vp, vp, i64, u64, u64, u64, u64, f32]
        lib.synth_gather_bf16.restype = None
        lib.synth_zero_experts.argtypes = [vp, ctypes.c_int32, ctypes.c_int32, u64, u64]
        lib.synth_zero_experts.restype = None
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(DEV_LIB):
            raise RuntimeError(f"device generator not built: {DEV_LIB} (run synth.build())")
        lib = ctypes.CDLL(DEV_LIB)
        u64, i64 = ctypes.c_uint64, ctypes.c_int64
        lib.synth_dev_fill_bf16.argtypes = [ctypes.c_void_p, i64, u64, u64, u64, u64, u64,
                                            ctypes.c_float, ctypes.c_void_p]
        lib.synth_dev_fill_bf16.restype = ctypes.c_int
        _dev = lib
    return _dev


def splitmix64(x: int) -> int:
    return int(_host_lib().synth_splitmix64(x & 0xFFFFFFFFFFFFFFFF))


def sigma_scale(sigma: float) -> float:
    return float(_host_lib().synth_sigma_scale(sigma))


def fill_bf16(n: int, seed: int, stream: int, rank: int, param: int, sigma: float,
              idx0: int = 0) -> np.ndarray:
    """n bf16 values (as uint16 bit patterns) at indices idx0 .. idx0+n-1."""
    out = np.empty(int(n), dtype=np.uint16)
    if n > 0:
        _host_lib().synth_fill_bf16(out.ctypes.data, int(n), int(idx0), seed, stream, rank,
                                    param, sigma_scale(sigma))
    return out


def gather_bf16(idx, seed: int, stream: int, rank: int, param: int, sigma: float) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(idx.size, dtype=np.uint16)
    if idx.size:
        _host_lib().synth_gather_bf16(out.ctypes.data, idx.ctypes.data, idx.size, seed, stream,
                                      rank, param, sigma_scale(sigma))
    return out


def zero_experts(n_experts: int, n_zero: int, seed: int, rank: int) -> np.ndarray:
    mask = np.zeros(n_experts, dtype=np.uint8)
    if n_experts:
        _host_lib().synth_zero_experts(mask.ctypes.data, n_experts, n_zero, seed, rank)
    return mask.astype(bool)


def zero_grad_params(group, seed: int, rank: int) -> set:
    """Param indices whose gradient is exactly zero on this rank (unrouted experts)."""
    if not group.n_experts:
        return set()
    mask = zero_experts(group.n_experts, group.n_zero_experts, seed, rank)
    out = set()
    for e in np.nonzero(mask)[0]:
        out.update(group.zero_expert_params[int(e)])
    return out


def grad_host(group, seed: int, rank: int, param: int) -> np.ndarray:
    """Rank `rank`'s unpadded gradient of param `param`, flat bf16 bits."""
    n = group.numel(param)
    if param in zero_grad_params(group, seed, rank):
        return np.zeros(n, dtype=np.uint16)
    return fill_bf16(n, seed, STREAM_GRAD, rank, param, group.grad_sigma)


def grads_host(group, seed: int) -> list:
    """grads[k][i]: every rank's unpadded per-parameter gradients."""
    out = []
    for k in range(group.world):
        zero = zero_grad_params(group, seed, k)
        row = []
        for i in range(group.n_params):
            n = group.numel(i)
            row.append(np.zeros(n, dtype=np.uint16) if i in zero else
                       fill_bf16(n, seed, STREAM_GRAD, k, i, group.grad_sigma))
        out.append(row)
    return out


def ag_host(group, shard_numel: int, seed: int) -> np.ndarray:
    """A rank-major all-gather buffer [W][shard_numel]: rank r's values at positions 0..Ns-1.

    Every position gets a value, pads included; placement must never read a pad.
    """
    W = group.world
    out = np.empty((W, int(shard_numel)), dtype=np.uint16)
    for r in range(W):
        out[r] = fill_bf16(shard_numel, seed, STREAM_AG, r, 0, group.param_sigma)
    return out


def dev_fill_bf16(tensor, seed: int, stream: int, rank: int, param: int, sigma: float,
                  idx0: int = 0, cuda_stream=None) -> None:
    """Fill a contiguous CUDA tensor (any 2-byte dtype) with the generator's values."""
    import torch
    assert tensor.is_cuda and tensor.is_contiguous() and tensor.element_size() == 2
    if cuda_stream is None:
        cuda_stream = torch.cuda.current_stream(tensor.device).cuda_stream
    rc = _dev_lib().synth_dev_fill_bf16(tensor.data_ptr(), tensor.numel(), int(idx0), seed,
                                        stream, rank, param, sigma_scale(sigma), cuda_stream)
    if rc != 0:
        raise RuntimeError(f"synth_dev_fill_bf16 failed with cudaError {rc}")


def dev_grads(group, seed: int, device="cuda") -> list:
    """grads[k][i] as separate device tensors (bf16), filled on the device."""
    import torch
    out = []
    for k in range(group.world):
        zero = zero_grad_params(group, seed, k)
        row = []
        for i in range(group.n_params):
            t = torch.empty(group.shapes[i], dtype=torch.bfloat16, device=device)
            if i in zero:
                t.zero_()
            else:
                dev_fill_bf16(t, seed, STREAM_GRAD, k, i, group.grad_sigma)
            row.append(t)
        out.append(row)
    return out


def dev_ag(group, shard_numel: int, seed: int, device="cuda"):
    """The rank-major all-gather buffer [W][Ns] on the device (same values as ag_host)."""
    import torch
    t = torch.empty((group.world, int(shard_numel)), dtype=torch.bfloat16, device=device)
    for r in range(group.world):
        dev_fill_bf16(t[r], seed, STREAM_AG, r, 0, group.param_sigma)
    return t
