"""The data-parallel exchange with one process per GPU: peers' buffers in the pointer tables.

In a data-parallel job each rank owns its gradients and its shard.  TIDE-RS has rank r reduce
its own shard from chunk r of every rank's gradients, and TIDE-AG has every rank place every
rank's shard into its own parameter storage (weekinpapers.com, Abstract; kongchang.com, "TIDE's
Design Approach").  Here the W ranks of a group are spread over n processes, one per GPU, W/n
consecutive ranks each.  A process keeps its ranks' gradients in one buffer (the gradient
arena) and their all-gather shards in another (the shard arena), laid out identically in every
process.  It exports both through CUDA IPC (tide_ipc_export); every other process maps them on
its own GPU (tide_ipc_open, which enables peer access, over NVLink on B200 systems), and the
mapped addresses go into the pointer tables that tide_rs_reduce and tide_ag_gather_place read.
The kernels then load peers' bytes like local ones.

This module is host-side plumbing only: arena layout, handle exchange over torch.distributed,
mapping, and table assembly.  No byte of the collectives moves here.  Nothing waits on another
process's GPU: the caller orders the ranks with host barriers (every rank's arenas are filled
before any rank reads them; no rank frees or unmaps while a peer may still read).
"""
from __future__ import annotations

from dataclasses import dataclass

from . import tide as T

ALIGN_ELEMS = 128   # 256 bytes of bf16: every param and shard starts on a 256-byte boundary


def ranks_of(proc: int, world: int, n_procs: int) -> range:
    """The group ranks held by process `proc`: W/n consecutive ranks."""
    if n_procs < 1 or world % n_procs != 0 or not 0 <= proc < n_procs:
        raise ValueError(f"{world} ranks cannot be spread evenly over {n_procs} processes")
    per = world // n_procs
    return range(proc * per, (proc + 1) * per)


def owner_of(rank: int, world: int, n_procs: int) -> int:
    """The process that holds group rank `rank`."""
    return rank // (world // n_procs)


def _align(n: int) -> int:
    return (n + ALIGN_ELEMS - 1) // ALIGN_ELEMS * ALIGN_ELEMS


@dataclass(frozen=True)
class ArenaLayout:
    """Element offsets inside a process's arenas (the same in every process).

    Gradient arena: for the process's j-th rank, param i's unpadded gradient at
    j * grad_stride + grad_off[i].  Shard arena: the j-th rank's bf16 [Ns] shard at
    j * shard_stride."""
    numel: tuple
    grad_off: tuple
    grad_stride: int
    shard_numel: int
    shard_stride: int
    per_proc: int

    @property
    def grad_elems(self) -> int:
        return self.per_proc * self.grad_stride

    @property
    def shard_elems(self) -> int:
        return self.per_proc * self.shard_stride


def arena_layout(shapes, world: int, n_procs: int, shard_numel: int) -> ArenaLayout:
    numel, off, acc = [], [], 0
    for s in shapes:
        n = 1
        for d in s:
            n *= int(d)
        numel.append(n)
        off.append(acc)
        acc += _align(n)
    per = world // n_procs
    return ArenaLayout(tuple(numel), tuple(off), max(acc, ALIGN_ELEMS), int(shard_numel),
                       _align(max(int(shard_numel), 1)), per)


def grad_table(layout: ArenaLayout, world: int, n_procs: int, grad_base) -> tuple:
    """(pointers, numels) of the W*P gradient table, index k*P + i, given every process's
    gradient arena address as seen from this process (grad_base[p], bytes)."""
    P = len(layout.numel)
    ptrs, numels = [], []
    for k in range(world):
        p = owner_of(k, world, n_procs)
        j = k - p * layout.per_proc
        for i in range(P):
            ptrs.append(grad_base[p] + 2 * (j * layout.grad_stride + layout.grad_off[i]))
            numels.append(layout.numel[i])
    return ptrs, numels


def shard_table(layout: ArenaLayout, world: int, n_procs: int, shard_base) -> list:
    """Pointers of the W all-gather shards, given every process's shard arena address."""
    out = []
    for r in range(world):
        p = owner_of(r, world, n_procs)
        out.append(shard_base[p] + 2 * (r - p * layout.per_proc) * layout.shard_stride)
    return out


_MAPPED = {}   # (handle bytes, device) -> [base, users]: one mapping per peer allocation


def open_shared(handle: bytes, device: int):
    """tide_ipc_open, once per (allocation, device) in this process.  CUDA maps an IPC handle
    at most once per process and device, and the caching allocator may put buffers of several
    owners' objects (arenas of different parameter groups) in one allocation: later users of
    the same handle get the first mapping, counted."""
    key = (bytes(handle), int(device))
    ent = _MAPPED.get(key)
    if ent is not None:
        ent[1] += 1
        return T.TIDE_OK, ent[0]
    st, base = T.tide_ipc_open(handle, device)
    if st == T.TIDE_OK:
        _MAPPED[key] = [base, 1]
    return st, base


def close_shared(base: int, device: int) -> int:
    """Drop one user of a mapping made by open_shared; unmap it when none is left."""
    for key, ent in _MAPPED.items():
        if ent[0] == base and key[1] == device:
            ent[1] -= 1
            if ent[1] > 0:
                return T.TIDE_OK
            del _MAPPED[key]
            break
    return T.tide_ipc_close(base, device)


class PeerMaps:
    """The other processes' arenas mapped into this one, on this process's device.

    exports[p] is process p's {name: (handle bytes, byte offset)} as tide_ipc_export gave it;
    `local` maps name -> this process's own address.  An allocation exported under several
    names is opened once.  opener/closer default to open_shared/close_shared (tests pass
    fakes).
    """

    def __init__(self, exports, me: int, device: int, local: dict, opener=None, closer=None):
        self.device = device
        self._close = closer or close_shared
        open_fn = opener or open_shared
        self._bases = {}
        self.addr = {}
        try:
            for p, exp in enumerate(exports):
                for name, (handle, offset) in exp.items():
                    if p == me:
                        self.addr[(p, name)] = local[name]
                        continue
                    if handle not in self._bases:
                        st, base = open_fn(handle, device)
                        if st != T.TIDE_OK:
                            raise T.TideError(st, f"tide_ipc_open (process {p}, {name})")
                        self._bases[handle] = base
                    self.addr[(p, name)] = self._bases[handle] + offset
        except Exception:
            self.close()
            raise

    def bases(self, name: str, n_procs: int) -> list:
        return [self.addr[(p, name)] for p in range(n_procs)]

    def close(self) -> None:
        for base in self._bases.values():
            self._close(base, self.device)
        self._bases = {}


def export(tensors: dict) -> dict:
    """{name: (handle bytes, offset)} of this process's arenas (CUDA tensors)."""
    out = {}
    for name, t in tensors.items():
        st, handle, offset, _ = T.tide_ipc_export(t.data_ptr())
        if st != T.TIDE_OK:
            raise T.TideError(st, f"tide_ipc_export ({name})")
        out[name] = (handle, offset)
    return out


def all_exports(local_exports: dict, group=None) -> list:
    """Every process's exports, in process order (torch.distributed all_gather_object)."""
    import torch.distributed as dist
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, local_exports, group=group)
    return out
