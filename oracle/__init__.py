"""CPU oracle for the TIDE hot path: TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference arm may import this package.  The CUDA path (the
``fsdp2_layout_aware_b200`` package and its C-ABI library) shares no code with
it and must never route through it.

Two independent implementations:
  * ``tide_oracle.c`` (loaded here through ctypes): the stock FSDP2 pipeline
    written out -- pack each rank into a full-group fp32 rank-major buffer,
    then sum over ranks in order; all-gather copy-out with zeroed pad rows.
  * ``oracle_np.py``: the direct-index definition with no packed buffer.
They must agree bit for bit.  The readings of the pages they share are listed
at the top of ``tide_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import oracle_np  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(_HERE, "liboracle.so")
SRC = os.path.join(_HERE, "tide_oracle.c")

_lib = None


def build(verbose: bool = False) -> None:
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-o", LIB, SRC]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)


def _load():
    global _lib
    if _lib is None:
        # TIDE_ORACLE_LIB points the pins at a deliberately broken build of this
        # oracle (tests/test_oracle_mutants.py) to show that they catch it.
        path = os.environ.get("TIDE_ORACLE_LIB")
        if path is None:
            if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
                build()
            path = LIB
        lib = ctypes.CDLL(path)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        p64 = ctypes.POINTER(ctypes.c_int64)
        lib.orc_layout.argtypes = [i64, i64, vp, vp, vp, vp, vp, p64]
        lib.orc_layout.restype = ctypes.c_int
        for name in ("orc_ag_copyout", "orc_pack_f32", "orc_slot_stage"):
            getattr(lib, name).argtypes = [i64, i64, vp, vp, vp, vp]
            getattr(lib, name).restype = ctypes.c_int
        for name in ("orc_rs_reduce_f32", "orc_rs_reduce_slots_f32"):
            getattr(lib, name).argtypes = [i64, i64, vp, vp, vp, i32, vp]
            getattr(lib, name).restype = ctypes.c_int
        lib.orc_slot_stage_f32.argtypes = [i64, i64, vp, vp, vp, vp]
        lib.orc_slot_stage_f32.restype = ctypes.c_int
        for name in ("orc_rs_reduce", "orc_rs_reduce_slots", "orc_rs_reduce_tree"):
            getattr(lib, name).argtypes = [i64, i64, vp, vp, vp, i32, vp]
            getattr(lib, name).restype = ctypes.c_int
        lib.orc_exact_f64.argtypes = [i64, i64, vp, vp, vp, vp, vp]
        lib.orc_exact_f64.restype = ctypes.c_int
        lib.orc_locate.argtypes = [i64, i64, vp, vp, i64, i64, p64, p64]
        lib.orc_locate.restype = ctypes.c_int
        for name in ("orc_sum_ranks", "orc_sum_ranks_tree"):
            getattr(lib, name).argtypes = [i64, vp, i32]
            getattr(lib, name).restype = ctypes.c_float
        lib.orc_ag_source.argtypes = [i64, i64, vp, vp, i64, i64, p64]
        lib.orc_ag_source.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dims(shapes):
    d0 = np.array([s[0] for s in shapes], dtype=np.int64)
    inner = np.array([int(np.prod(s[1:], dtype=np.int64)) if len(s) > 1 else 1 for s in shapes],
                     dtype=np.int64)
    return d0, inner


def _ptrs(arrays):
    return (ctypes.c_void_p * max(1, len(arrays)))(*[a.ctypes.data for a in arrays])


class Layout:
    def __init__(self, S, c, off, Ns):
        self.S, self.c, self.off, self.Ns = S, c, off, Ns


def layout(world: int, shapes) -> Layout:
    d0, inner = _dims(shapes)
    P = len(shapes)
    S, c, off = (np.zeros(max(P, 1), dtype=np.int64) for _ in range(3))
    Ns = ctypes.c_int64(0)
    rc = _load().orc_layout(world, P, d0.ctypes.data, inner.ctypes.data, S.ctypes.data,
                            c.ctypes.data, off.ctypes.data, ctypes.byref(Ns))
    if rc != 0:
        raise ValueError("bad group")
    return Layout([int(x) for x in S[:P]], [int(x) for x in c[:P]], [int(x) for x in off[:P]],
                  int(Ns.value))


def rs_reduce(world: int, shapes, grads, scale_mode: int) -> np.ndarray:
    """grads[k][i]: contiguous uint16 arrays (bf16 bits).  Returns fp32 [W*Ns]."""
    d0, inner = _dims(shapes)
    P = len(shapes)
    Ns = layout(world, shapes).Ns
    out = np.empty(world * Ns, dtype=np.float32)
    flat = [np.ascontiguousarray(grads[k][i], dtype=np.uint16) for k in range(world) for i in range(P)]
    rc = _load().orc_rs_reduce(world, P, d0.ctypes.data, inner.ctypes.data, _ptrs(flat),
                               scale_mode, out.ctypes.data)
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return out


def rs_reduce_tree(world: int, shapes, grads, scale_mode: int) -> np.ndarray:
    """The reduce-scatter in tree order (pairs level by level, odd one carried).  fp32 [W*Ns]."""
    d0, inner = _dims(shapes)
    P = len(shapes)
    Ns = layout(world, shapes).Ns
    out = np.empty(world * Ns, dtype=np.float32)
    flat = [np.ascontiguousarray(grads[k][i], dtype=np.uint16) for k in range(world) for i in range(P)]
    rc = _load().orc_rs_reduce_tree(world, P, d0.ctypes.data, inner.ctypes.data, _ptrs(flat),
                                    scale_mode, out.ctypes.data)
    if rc != 0:
        raise MemoryError("oracle allocation failed")
    return out


def pack_f32(world: int, shapes, g_rank) -> np.ndarray:
    d0, inner = _dims(shapes)
    Ns = layout(world, shapes).Ns
    buf = np.empty(world * Ns, dtype=np.float32)
    g = [np.ascontiguousarray(x, dtype=np.uint16) for x in g_rank]
    _load().orc_pack_f32(world, len(shapes), d0.ctypes.data, inner.ctypes.data, _ptrs(g),
                         buf.ctypes.data)
    return buf


def ag_copyout(world: int, shapes, ag: np.ndarray) -> list:
    """ag: uint16 [W*Ns].  Returns the padded per-param storage (flat uint16 arrays)."""
    d0, inner = _dims(shapes)
    L = layout(world, shapes)
    ag = np.ascontiguousarray(ag, dtype=np.uint16).reshape(-1)
    assert ag.size == world * L.Ns
    params = [np.full(world * L.c[i], 0xBEEF, dtype=np.uint16) for i in range(len(shapes))]
    _load().orc_ag_copyout(world, len(shapes), d0.ctypes.data, inner.ctypes.data, ag.ctypes.data,
                           _ptrs(params))
    return params


def slot_stage(world: int, shapes, g_rank, slot: np.ndarray) -> None:
    """Stage one rank's grads into `slot` (uint16 [W*Ns]) in place; pads untouched."""
    d0, inner = _dims(shapes)
    g = [np.ascontiguousarray(x, dtype=np.uint16) for x in g_rank]
    assert slot.dtype == np.uint16 and slot.flags.c_contiguous
    _load().orc_slot_stage(world, len(shapes), d0.ctypes.data, inner.ctypes.data, _ptrs(g),
                           slot.ctypes.data)


def rs_reduce_slots(world: int, shapes, slots, scale_mode: int) -> np.ndarray:
    d0, inner = _dims(shapes)
    Ns = layout(world, shapes).Ns
    out = np.empty(world * Ns, dtype=np.float32)
    sl = [np.ascontiguousarray(s, dtype=np.uint16).reshape(-1) for s in slots]
    _load().orc_rs_reduce_slots(world, len(shapes), d0.ctypes.data, inner.ctypes.data, _ptrs(sl),
                                scale_mode, out.ctypes.data)
    return out


def rs_reduce_f32(world: int, shapes, grads, scale_mode: int) -> np.ndarray:
    """rs_reduce for fp32 gradients: grads[k][i] contiguous float32 arrays (or their uint32
    bits).  Returns fp32 [W*Ns]."""
    d0, inner = _dims(shapes)
    P = len(shapes)
    Ns = layout(world, shapes).Ns
    out = np.empty(world * Ns, dtype=np.float32)
    flat = [np.ascontiguousarray(grads[k][i]).reshape(-1).view(np.float32)
            for k in range(world) for i in range(P)]
    _load().orc_rs_reduce_f32(world, P, d0.ctypes.data, inner.ctypes.data, _ptrs(flat),
                              scale_mode, out.ctypes.data)
    return out


def slot_stage_f32(world: int, shapes, g_rank, slot: np.ndarray) -> None:
    """Stage one rank's fp32 grads into `slot` ([W*Ns] of 4-byte words: float32 or uint32) in
    place, as a copy of the words; pads untouched."""
    d0, inner = _dims(shapes)
    g = [np.ascontiguousarray(x).reshape(-1).view(np.uint32) for x in g_rank]
    assert slot.dtype.itemsize == 4 and slot.flags.c_contiguous
    _load().orc_slot_stage_f32(world, len(shapes), d0.ctypes.data, inner.ctypes.data, _ptrs(g),
                               slot.ctypes.data)


def rs_reduce_slots_f32(world: int, shapes, slots, scale_mode: int) -> np.ndarray:
    """Slot-Reuse phase 2 over fp32 slots ([W*Ns] each, float32 or their uint32 bits)."""
    d0, inner = _dims(shapes)
    Ns = layout(world, shapes).Ns
    out = np.empty(world * Ns, dtype=np.float32)
    sl = [np.ascontiguousarray(s).reshape(-1).view(np.float32) for s in slots]
    _load().orc_rs_reduce_slots_f32(world, len(shapes), d0.ctypes.data, inner.ctypes.data,
                                    _ptrs(sl), scale_mode, out.ctypes.data)
    return out


def exact_f64(world: int, shapes, grads):
    """(E, A): exact fp64 sums and sums of magnitudes, [W*Ns] each."""
    d0, inner = _dims(shapes)
    P = len(shapes)
    Ns = layout(world, shapes).Ns
    E = np.empty(world * Ns, dtype=np.float64)
    A = np.empty(world * Ns, dtype=np.float64)
    flat = [np.ascontiguousarray(grads[k][i], dtype=np.uint16) for k in range(world) for i in range(P)]
    _load().orc_exact_f64(world, P, d0.ctypes.data, inner.ctypes.data, _ptrs(flat),
                          E.ctypes.data, A.ctypes.data)
    return E, A


def locate(world: int, shapes, r: int, j: int):
    """(status, param, src_idx) for position j of rank r's shard: 1 valid, 0 pad, -1 outside."""
    d0, inner = _dims(shapes)
    p, s = ctypes.c_int64(-1), ctypes.c_int64(-1)
    st = _load().orc_locate(world, len(shapes), d0.ctypes.data, inner.ctypes.data, r, j,
                            ctypes.byref(p), ctypes.byref(s))
    return int(st), int(p.value), int(s.value)


def sum_ranks(vals, scale_mode: int) -> np.float32:
    v = np.ascontiguousarray(vals, dtype=np.uint16)
    return np.float32(_load().orc_sum_ranks(v.size, v.ctypes.data, scale_mode))


def sum_ranks_tree(vals, scale_mode: int) -> np.float32:
    v = np.ascontiguousarray(vals, dtype=np.uint16)
    return np.float32(_load().orc_sum_ranks_tree(v.size, v.ctypes.data, scale_mode))


def ag_source(world: int, shapes, i: int, q: int):
    """(status, ag_idx) for element q of param i's padded storage."""
    d0, inner = _dims(shapes)
    a = ctypes.c_int64(-1)
    st = _load().orc_ag_source(world, len(shapes), d0.ctypes.data, inner.ctypes.data, i, q,
                               ctypes.byref(a))
    return int(st), int(a.value)
