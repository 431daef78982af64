"""ctypes binding of libtide.so (include/tide.h): argument marshalling only.

Each ``tide_*`` function here has the C entry point's name and arguments, with
Python ints for pointers and sizes; every step of the work runs in the
library's CUDA kernels or copy-engine calls.  If the library has not been
built the import fails loudly: there is no fallback path.

``Plan`` is a thin convenience wrapper that takes torch tensors (device memory
and the current CUDA stream come from PyTorch) and forwards their pointers.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtide.so")

TIDE_OK = 0
TIDE_ERR_INVALID_ARG = -1
TIDE_ERR_ALIGNMENT = -2
TIDE_ERR_SIZE = -3
TIDE_ERR_CUDA = -4
TIDE_ERR_NOMEM = -5
TIDE_ERR_DEVICE = -6
TIDE_ERR_KERNEL_CHECK = -7

TIDE_ENGINE_SM = 0
TIDE_ENGINE_CE = 1
TIDE_ORDER_RANK = 0
TIDE_ORDER_TREE = 1
TIDE_SCALE_NONE = 0
TIDE_SCALE_INV_WORLD = 1
TIDE_PLAN_HOST_ONLY = 1
TIDE_PLAN_TMA = 2
TIDE_PLAN_TEST_TMA_TIMEOUT = 4
TIDE_PLAN_SHORT_CTAS = 8
TIDE_KCHECK_TILE, TIDE_KCHECK_TIMEOUT = 1, 2
TIDE_MAX_WORLD = 256
TIDE_TILE_ELEMS = 8192
TIDE_NOALLOC_SCRATCH_BYTES = 1 << 20
TIDE_IPC_HANDLE_BYTES = 64

(K_RS, K_AG, K_STAGE, K_SLOT_RS, K_RS_TMA, K_SLOT_RS_TMA, K_RS_V32, K_SLOT_RS_V32, K_RS_TREE,
 K_SLOT_RS_TREE, K_AG_GATHER, K_RS_TREE_V32, K_SLOT_RS_TREE_V32) = range(13)
KERNEL_NAMES = ("rs", "ag", "stage", "slot_rs", "rs_tma", "slot_rs_tma", "rs_v32", "slot_rs_v32",
                "rs_tree", "slot_rs_tree", "ag_gather", "rs_tree_v32", "slot_rs_tree_v32",
                "stage_f32", "slot_rs_f32", "rs_f32")


class tide_param_t(ctypes.Structure):
    _fields_ = [("dim0", ctypes.c_int64), ("inner", ctypes.c_int64)]


class tide_tile_t(ctypes.Structure):
    _fields_ = [("src_off", ctypes.c_int64), ("dst_off", ctypes.c_int64),
                ("param", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("n_valid", ctypes.c_int32), ("n_total", ctypes.c_int32)]


class TideError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {tide_status_string(status)} ({status})")


_lib = None

_i32, _i64, _u32, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p
_P = ctypes.POINTER

_SIGNATURES = {
    "tide_plan_group": (_i32, [_P(tide_param_t), _i32, _i32, _i32, _u32, _P(_vp)]),
    "tide_plan_group_rank": (_i32, [_P(tide_param_t), _i32, _i32, _i32, _i32, _u32, _P(_vp)]),
    "tide_ag_gather_place": (_i32, [_vp, _P(_vp), _i64, _P(_vp), _P(_i64), _i32, _i32, _vp]),
    "tide_plan_destroy": (None, [_vp]),
    "tide_plan_info": (_i32, [_vp, _P(_i32), _P(_i32), _P(_i64), _P(_i64), _P(_i64)]),
    "tide_plan_query": (_i32, [_vp, _i32, _P(_i64), _P(_i64), _P(_i64), _P(_i64)]),
    "tide_plan_tiles": (_i32, [_vp, _P(tide_tile_t), _i64, _P(_i64)]),
    "tide_ag_place": (_i32, [_vp, _vp, _i64, _P(_vp), _P(_i64), _i32, _i32, _vp]),
    "tide_rs_reduce": (_i32, [_vp, _P(_vp), _P(_i64), _vp, _i64, _i32, _i32, _P(_vp), _i64,
                              _i32, _i32, _vp]),
    "tide_rs_stage": (_i32, [_vp, _P(_vp), _P(_i64), _P(_vp), _i64, _i32, _i32, _vp]),
    "tide_flag_signal": (_i32, [_vp, ctypes.c_uint32, _vp]),
    "tide_flag_wait": (_i32, [_P(_vp), _i32, ctypes.c_uint32, _i64, _vp, _vp]),
    "tide_rs_stage_one": (_i32, [_vp, _P(_vp), _P(_i64), _vp, _i64, _i32, _i32, _vp]),
    "tide_rs_reduce_slots": (_i32, [_vp, _P(_vp), _i64, _vp, _i64, _i32, _i32, _i32, _vp]),
    "tide_rs_stage_one_f32": (_i32, [_vp, _P(_vp), _P(_i64), _vp, _i64, _i32, _i32, _vp]),
    "tide_rs_reduce_slots_f32": (_i32, [_vp, _P(_vp), _i64, _vp, _i64, _i32, _i32, _vp]),
    "tide_rs_reduce_f32": (_i32, [_vp, _P(_vp), _P(_i64), _vp, _i64, _i32, _i32, _vp]),
    "tide_rs_reduce_noalloc": (_i32, [_P(tide_param_t), _i32, _i32, _P(_vp), _P(_i64), _vp, _i64,
                                      _i32, _i32, _vp]),
    "tide_rs_reduce_pipelined": (_i32, [_vp, _P(_vp), _P(_i64), _vp, _i64, _i32, _i32, _P(_vp),
                                        _i64, _i32, _i32, _vp, _vp]),
    "tide_plan_check": (_i32, [_vp, _vp]),
    "tide_plan_errors": (_i32, [_vp, _vp, _P(_i32)]),
    "tide_launch_ctas": (_i32, [_vp, _i32, _i32, _P(_i32)]),
    "tide_plan_last_launch": (_i32, [_vp, _P(_i32), _P(_i32)]),
    "tide_ipc_export": (_i32, [_vp, _vp, _P(_i64), _P(_i32)]),
    "tide_ipc_open": (_i32, [_vp, _i32, _P(_vp)]),
    "tide_ipc_close": (_i32, [_vp, _i32]),
    "tide_peer_access": (_i32, [_i32, _i32, _P(_i32)]),
    "tide_status_string": (ctypes.c_char_p, [_i32]),
    "tide_abi_version": (_i32, []),
}


def lib():
    """The loaded libtide.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtide.so is not built ({LIB_PATH}); run "
                               "`python -m fsdp2_layout_aware_b200.build` (there is no CPU fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _ptr_array(ptrs):
    """A ctypes void* array of the given addresses (an existing ctypes array passes through)."""
    if isinstance(ptrs, ctypes.Array):
        return ptrs
    return (_vp * max(1, len(ptrs)))(*ptrs)


def _i64_array(vals):
    if isinstance(vals, ctypes.Array):
        return vals
    return (_i64 * max(1, len(vals)))(*[int(v) for v in vals])


class TensorTable:
    """Device pointers and element counts of a fixed list of tensors, marshalled once.

    Passing one to the Plan methods in place of a list skips the per-call
    collection of pointers and sizes (for a group of 393 params at W=8 that is
    3144 tensors).  The table holds references to the tensors; their storage
    must not be replaced while the table is in use.
    """

    def __init__(self, tensors):
        self.tensors = list(tensors)
        self.ptrs = _ptr_array([t.data_ptr() for t in self.tensors])
        self.numels = _i64_array([t.numel() for t in self.tensors])
        self.min_numel = min((t.numel() for t in self.tensors), default=0)

    def __len__(self):
        return len(self.tensors)


class PointerTable(TensorTable):
    """A table of raw device addresses and element counts (for example peers' buffers mapped
    through tide_ipc_open), usable wherever the Plan methods accept a TensorTable.  `keep`
    holds references to whatever owns the memory."""

    def __init__(self, ptrs, numels, keep=()):
        self.tensors = list(keep)
        self.ptrs = _ptr_array([int(p) for p in ptrs])
        self.numels = _i64_array(numels)
        self.min_numel = min((int(n) for n in numels), default=0)
        self._n = len(ptrs)

    def __len__(self):
        return self._n


def _table(tensors) -> TensorTable:
    """A TensorTable as is, or one built now from a (possibly nested per rank) list."""
    if isinstance(tensors, TensorTable):
        return tensors
    flat = [t for row in tensors for t in row] if tensors and isinstance(tensors[0], (list, tuple)) \
        else list(tensors)
    return TensorTable(flat)


def _require_f32(table, *tensors) -> None:
    """The C calls of fp32 buffers count 4-byte elements: refuse torch tensors of another
    dtype (a PointerTable's raw addresses carry none and are taken as they are)."""
    import torch
    held = [] if isinstance(table, PointerTable) else list(table.tensors)
    for t in held + list(tensors):
        if t.dtype != torch.float32:
            raise TypeError(f"fp32 buffer expected, got {t.dtype}")


def _check(status: int, where: str) -> None:
    if status != TIDE_OK:
        raise TideError(status, where)


# --------------------------------------------------------------------------- C-ABI mirrors


def tide_status_string(status: int) -> str:
    return lib().tide_status_string(status).decode()


def tide_abi_version() -> int:
    return lib().tide_abi_version()


def tide_plan_group(params, world: int, device: int, flags: int = 0):
    """params: sequence of (dim0, inner).  Returns (status, plan handle or None)."""
    arr = (tide_param_t * max(1, len(params)))()
    for j, (d0, inner) in enumerate(params):
        arr[j].dim0, arr[j].inner = int(d0), int(inner)
    out = _vp()
    st = lib().tide_plan_group(arr, len(params), world, device, flags, ctypes.byref(out))
    return st, (out.value if st == TIDE_OK else None)


def tide_plan_group_rank(params, world: int, rank: int, device: int, flags: int = 0):
    """A plan for one output rank.  Returns (status, plan handle or None)."""
    arr = (tide_param_t * max(1, len(params)))()
    for j, (d0, inner) in enumerate(params):
        arr[j].dim0, arr[j].inner = int(d0), int(inner)
    out = _vp()
    st = lib().tide_plan_group_rank(arr, len(params), world, rank, device, flags, ctypes.byref(out))
    return st, (out.value if st == TIDE_OK else None)


def tide_plan_destroy(plan) -> None:
    lib().tide_plan_destroy(plan)


def tide_plan_info(plan):
    w, p = _i32(), _i32()
    ns, nt, ws = _i64(), _i64(), _i64()
    st = lib().tide_plan_info(plan, ctypes.byref(w), ctypes.byref(p), ctypes.byref(ns),
                              ctypes.byref(nt), ctypes.byref(ws))
    return st, dict(world=w.value, n_params=p.value, shard_numel=ns.value, n_tiles=nt.value,
                    workspace_bytes=ws.value)


def tide_plan_query(plan, param: int):
    a, b, c, d = _i64(), _i64(), _i64(), _i64()
    st = lib().tide_plan_query(plan, param, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c),
                               ctypes.byref(d))
    return st, dict(shard_rows=a.value, shard_offset=b.value, padded_numel=c.value,
                    chunk_numel=d.value)


def tide_plan_tiles(plan, capacity: int):
    arr = (tide_tile_t * max(1, capacity))()
    n = _i64()
    st = lib().tide_plan_tiles(plan, arr, capacity, ctypes.byref(n))
    return st, arr[: n.value]


def tide_ag_place(plan, ag_buf: int, ag_numel: int, param_storage, param_numel, engine: int,
                  max_ctas: int, stream: int) -> int:
    return lib().tide_ag_place(plan, ag_buf, ag_numel, _ptr_array(param_storage),
                               _i64_array(param_numel), engine, max_ctas, stream)


def tide_ag_gather_place(plan, shards, shard_numel: int, param_storage, param_numel, engine: int,
                         max_ctas: int, stream: int) -> int:
    return lib().tide_ag_gather_place(plan, _ptr_array(shards), shard_numel, _ptr_array(param_storage),
                                      _i64_array(param_numel), engine, max_ctas, stream)


def tide_rs_reduce(plan, grads, grad_numel, out: int, out_numel: int, scale_mode: int, order: int,
                   slots, slot_numel: int, engine: int, max_ctas: int, stream: int) -> int:
    slot_arr = _ptr_array(slots) if slots is not None else None
    return lib().tide_rs_reduce(plan, _ptr_array(grads), _i64_array(grad_numel), out, out_numel,
                                scale_mode, order, slot_arr, slot_numel, engine, max_ctas, stream)


def tide_rs_stage(plan, grads, grad_numel, slots, slot_numel: int, engine: int, max_ctas: int,
                  stream: int) -> int:
    slot_arr = _ptr_array(slots) if slots is not None else None
    return lib().tide_rs_stage(plan, _ptr_array(grads), _i64_array(grad_numel), slot_arr,
                               slot_numel, engine, max_ctas, stream)


def tide_flag_signal(flag: int, value: int, stream: int = 0) -> int:
    """Store `value` into the device flag at `flag` after every earlier write of this device
    (stream-ordered, release semantics at system scope)."""
    return lib().tide_flag_signal(flag, value & 0xFFFFFFFF, stream)


def tide_flag_wait(flags, value: int, timeout_ns: int, status: int, stream: int = 0) -> int:
    """One kernel that polls the device flags until each reaches epoch `value` or timeout_ns
    passes, then writes the int32 at `status`: 0, or 1 + the first late flag's index."""
    return lib().tide_flag_wait(_ptr_array(flags), len(flags), value & 0xFFFFFFFF, timeout_ns,
                                status, stream)


def tide_rs_stage_one(plan, grads, grad_numel, slot: int, slot_numel: int, engine: int,
                      max_ctas: int, stream: int) -> int:
    return lib().tide_rs_stage_one(plan, _ptr_array(grads), _i64_array(grad_numel), slot, slot_numel,
                                   engine, max_ctas, stream)


def tide_rs_reduce_slots(plan, slots, slot_numel: int, out: int, out_numel: int, scale_mode: int,
                         order: int, max_ctas: int, stream: int) -> int:
    slot_arr = _ptr_array(slots) if slots is not None else None
    return lib().tide_rs_reduce_slots(plan, slot_arr, slot_numel, out, out_numel, scale_mode,
                                      order, max_ctas, stream)


def tide_rs_stage_one_f32(plan, grads, grad_numel, slot: int, slot_numel: int, engine: int,
                          max_ctas: int, stream: int) -> int:
    return lib().tide_rs_stage_one_f32(plan, _ptr_array(grads), _i64_array(grad_numel), slot,
                                       slot_numel, engine, max_ctas, stream)


def tide_rs_reduce_f32(plan, grads, grad_numel, out: int, out_numel: int, scale_mode: int,
                       max_ctas: int, stream: int) -> int:
    return lib().tide_rs_reduce_f32(plan, _ptr_array(grads), _i64_array(grad_numel), out, out_numel,
                                    scale_mode, max_ctas, stream)


def tide_rs_reduce_slots_f32(plan, slots, slot_numel: int, out: int, out_numel: int, scale_mode: int,
                             max_ctas: int, stream: int) -> int:
    slot_arr = _ptr_array(slots) if slots is not None else None
    return lib().tide_rs_reduce_slots_f32(plan, slot_arr, slot_numel, out, out_numel, scale_mode,
                                          max_ctas, stream)


def tide_rs_reduce_noalloc(params, world: int, grads, grad_numel, out: int, out_numel: int,
                           scale_mode: int, max_ctas: int, stream: int) -> int:
    """params: sequence of (dim0, inner); grads: W*P device pointers, index k*P + i."""
    arr = (tide_param_t * max(1, len(params)))()
    for j, (d0, inner) in enumerate(params):
        arr[j].dim0, arr[j].inner = int(d0), int(inner)
    return lib().tide_rs_reduce_noalloc(arr, len(params), world, _ptr_array(grads),
                                        _i64_array(grad_numel), out, out_numel, scale_mode,
                                        max_ctas, stream)


def tide_rs_reduce_pipelined(plan, grads, grad_numel, out: int, out_numel: int, scale_mode: int,
                             order: int, slots, slot_numel: int, n_segments: int, max_ctas: int,
                             stream: int, copy_stream: int) -> int:
    slot_arr = _ptr_array(slots) if slots is not None else None
    return lib().tide_rs_reduce_pipelined(plan, _ptr_array(grads), _i64_array(grad_numel), out,
                                          out_numel, scale_mode, order, slot_arr, slot_numel,
                                          n_segments, max_ctas, stream, copy_stream)


def tide_plan_check(plan, stream: int) -> int:
    return lib().tide_plan_check(plan, stream)


def tide_plan_errors(plan, stream: int):
    bits = ctypes.c_int32(0)
    st = lib().tide_plan_errors(plan, stream, ctypes.byref(bits))
    return st, bits.value


def tide_plan_last_launch(plan):
    k, n = _i32(), _i32()
    st = lib().tide_plan_last_launch(plan, ctypes.byref(k), ctypes.byref(n))
    return st, k.value, n.value


def tide_launch_ctas(plan, kernel: int, max_ctas: int):
    n = _i32()
    st = lib().tide_launch_ctas(plan, kernel, max_ctas, ctypes.byref(n))
    return st, n.value


def tide_ipc_export(dev_ptr: int):
    """(status, handle bytes, offset, device) of the allocation holding dev_ptr."""
    h = ctypes.create_string_buffer(TIDE_IPC_HANDLE_BYTES)
    off, dev = _i64(0), _i32(-1)
    st = lib().tide_ipc_export(dev_ptr, h, ctypes.byref(off), ctypes.byref(dev))
    return st, h.raw, off.value, dev.value


def tide_ipc_open(handle: bytes, device: int):
    """(status, base pointer) of another process's exported allocation, mapped for `device`."""
    if len(handle) != TIDE_IPC_HANDLE_BYTES:
        return TIDE_ERR_INVALID_ARG, 0
    h = ctypes.create_string_buffer(handle, TIDE_IPC_HANDLE_BYTES)
    base = _vp(0)
    st = lib().tide_ipc_open(h, device, ctypes.byref(base))
    return st, base.value or 0


def tide_ipc_close(base: int, device: int) -> int:
    return lib().tide_ipc_close(base, device)


def tide_peer_access(device: int, peer: int):
    v = _i32(0)
    st = lib().tide_peer_access(device, peer, ctypes.byref(v))
    return st, v.value


# --------------------------------------------------------------------------- torch convenience


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


class Plan:
    """A parameter group over `world` simulated ranks, planned on one device.

    shapes: parameter shapes (dim 0 first).  Tensors passed to the methods are
    only read for their data pointers and sizes.
    """

    def __init__(self, shapes, world: int, device=None, host_only: bool = False,
                 tma: bool = False, test_tma_timeout: bool = False, rank=None,
                 short_ctas: bool = False):
        """rank: None for the whole group (all W output shards), or one output rank r, whose
        rs_reduce then writes only its own [Ns] shard.  short_ctas: one short-lived CTA per
        unit of work instead of a persistent grid (TIDE_PLAN_SHORT_CTAS)."""
        self.shapes = [tuple(int(d) for d in s) for s in shapes]
        self.world = int(world)
        if host_only:
            dev = 0
        else:
            import torch
            dev = torch.cuda.current_device() if device is None else torch.device(device).index
            dev = 0 if dev is None else dev
        params = [(s[0], _prod(s[1:])) for s in self.shapes]
        flags = ((TIDE_PLAN_HOST_ONLY if host_only else 0) | (TIDE_PLAN_TMA if tma else 0) |
                 (TIDE_PLAN_TEST_TMA_TIMEOUT if test_tma_timeout else 0) |
                 (TIDE_PLAN_SHORT_CTAS if short_ctas else 0))
        self.rank = None if rank is None else int(rank)
        if self.rank is None:
            st, handle = tide_plan_group(params, self.world, dev, flags)
        else:
            st, handle = tide_plan_group_rank(params, self.world, self.rank, dev, flags)
        _check(st, "tide_plan_group")
        self.handle = handle
        self.device_index = dev
        st, info = tide_plan_info(handle)
        _check(st, "tide_plan_info")
        self.shard_numel = info["shard_numel"]
        self.n_tiles = info["n_tiles"]
        self.workspace_bytes = info["workspace_bytes"]
        self.n_params = info["n_params"]

    def close(self) -> None:
        if getattr(self, "handle", None):
            tide_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def query(self, param: int) -> dict:
        st, q = tide_plan_query(self.handle, param)
        _check(st, "tide_plan_query")
        return q

    def tiles(self):
        st, t = tide_plan_tiles(self.handle, self.n_tiles)
        _check(st, "tide_plan_tiles")
        return t

    def launch_ctas(self, kernel: int, max_ctas: int = 0) -> int:
        st, n = tide_launch_ctas(self.handle, kernel, max_ctas)
        _check(st, "tide_launch_ctas")
        return n

    def last_launch(self):
        """(kernel id, CTAs) of the most recent kernel launch on this plan."""
        st, k, n = tide_plan_last_launch(self.handle)
        _check(st, "tide_plan_last_launch")
        return k, n

    # grads: rank k's gradient of param i at grads[k][i], or a TensorTable of the W*P
    # gradients in that order; params and slots: a list or a TensorTable.

    def ag_place(self, ag, params, engine: int = TIDE_ENGINE_SM, max_ctas: int = 0,
                 stream=None) -> None:
        p = _table(params)
        st = tide_ag_place(self.handle, ag.data_ptr(), ag.numel(), p.ptrs, p.numels, engine,
                           max_ctas, _stream_handle(stream))
        _check(st, "tide_ag_place")

    def ag_gather_place(self, shards, params, engine: int = TIDE_ENGINE_SM, max_ctas: int = 0,
                        stream=None) -> None:
        """Place every rank's shard (shards[r]: bf16 [Ns], possibly a peer's memory)."""
        s, p = _table(shards), _table(params)
        st = tide_ag_gather_place(self.handle, s.ptrs, s.min_numel, p.ptrs, p.numels, engine,
                                  max_ctas, _stream_handle(stream))
        _check(st, "tide_ag_gather_place")

    def rs_reduce(self, grads, out, scale_mode: int = TIDE_SCALE_INV_WORLD,
                  order: int = TIDE_ORDER_RANK, slots=None, engine: int = TIDE_ENGINE_SM,
                  max_ctas: int = 0, stream=None) -> None:
        """grads[k][i]: rank k's gradient of param i; out: fp32 [W*Ns]."""
        g = _table(grads)
        s = None if slots is None else _table(slots)
        st = tide_rs_reduce(self.handle, g.ptrs, g.numels, out.data_ptr(), out.numel(), scale_mode,
                            order, None if s is None else s.ptrs, 0 if s is None else s.min_numel,
                            engine, max_ctas, _stream_handle(stream))
        _check(st, "tide_rs_reduce")

    def rs_stage(self, grads, slots, engine: int = TIDE_ENGINE_SM, max_ctas: int = 0,
                 stream=None) -> None:
        g, s = _table(grads), _table(slots)
        st = tide_rs_stage(self.handle, g.ptrs, g.numels, s.ptrs, s.min_numel, engine, max_ctas,
                           _stream_handle(stream))
        _check(st, "tide_rs_stage")

    def rs_stage_one(self, grads, slot, engine: int = TIDE_ENGINE_SM, max_ctas: int = 0,
                     stream=None) -> None:
        """One rank's P gradients into its own slot (bf16 [W][Ns])."""
        g = _table(grads)
        st = tide_rs_stage_one(self.handle, g.ptrs, g.numels, slot.data_ptr(), slot.numel(), engine,
                               max_ctas, _stream_handle(stream))
        _check(st, "tide_rs_stage_one")

    def rs_reduce_slots(self, slots, out, scale_mode: int = TIDE_SCALE_INV_WORLD,
                        order: int = TIDE_ORDER_RANK, max_ctas: int = 0, stream=None) -> None:
        """Every rank's shard from the W slots ([W][Ns] out); with a one-rank plan, that rank's
        shard ([Ns] out), the slots possibly peers' memory."""
        s = _table(slots)
        st = tide_rs_reduce_slots(self.handle, s.ptrs, s.min_numel, out.data_ptr(), out.numel(),
                                  scale_mode, order, max_ctas, _stream_handle(stream))
        _check(st, "tide_rs_reduce_slots")

    def rs_stage_one_f32(self, grads, slot, engine: int = TIDE_ENGINE_SM, max_ctas: int = 0,
                         stream=None) -> None:
        """One rank's P fp32 gradients into its own fp32 slot ([W][Ns])."""
        g = _table(grads)
        _require_f32(g, slot)
        st = tide_rs_stage_one_f32(self.handle, g.ptrs, g.numels, slot.data_ptr(), slot.numel(),
                                   engine, max_ctas, _stream_handle(stream))
        _check(st, "tide_rs_stage_one_f32")

    def rs_reduce_f32(self, grads, out, scale_mode: int = TIDE_SCALE_INV_WORLD, max_ctas: int = 0,
                      stream=None) -> None:
        """rs_reduce for fp32 gradients (grads[k][i], or a flat k*P + i table), rank order."""
        g = _table(grads)
        _require_f32(g, out)
        st = tide_rs_reduce_f32(self.handle, g.ptrs, g.numels, out.data_ptr(), out.numel(), scale_mode,
                                max_ctas, _stream_handle(stream))
        _check(st, "tide_rs_reduce_f32")

    def rs_reduce_slots_f32(self, slots, out, scale_mode: int = TIDE_SCALE_INV_WORLD,
                            max_ctas: int = 0, stream=None) -> None:
        """rs_reduce_slots over W fp32 slots (rank order)."""
        s = _table(slots)
        _require_f32(s, out)
        st = tide_rs_reduce_slots_f32(self.handle, s.ptrs, s.min_numel, out.data_ptr(), out.numel(),
                                      scale_mode, max_ctas, _stream_handle(stream))
        _check(st, "tide_rs_reduce_slots_f32")

    def rs_reduce_pipelined(self, grads, out, slots, n_segments: int, copy_stream,
                            scale_mode: int = TIDE_SCALE_INV_WORLD, order: int = TIDE_ORDER_RANK,
                            max_ctas: int = 0, stream=None) -> None:
        """Slot-Reuse with copy-engine staging on `copy_stream` overlapping the reduction."""
        g, s = _table(grads), _table(slots)
        st = tide_rs_reduce_pipelined(self.handle, g.ptrs, g.numels, out.data_ptr(), out.numel(),
                                      scale_mode, order, s.ptrs, s.min_numel, n_segments, max_ctas,
                                      _stream_handle(stream), _stream_handle(copy_stream))
        _check(st, "tide_rs_reduce_pipelined")

    def check(self, stream=None) -> None:
        _check(tide_plan_check(self.handle, _stream_handle(stream)), "tide_plan_check")

    def errors(self, stream=None) -> int:
        """Read and clear the device error word; its TIDE_KCHECK_* bits (0 if none)."""
        st, bits = tide_plan_errors(self.handle, _stream_handle(stream))
        if st not in (TIDE_OK, TIDE_ERR_KERNEL_CHECK):
            _check(st, "tide_plan_errors")
        return bits


def _prod(dims) -> int:
    n = 1
    for d in dims:
        n *= int(d)
    return n
