"""Second oracle: the direct-index definition, in numpy.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Where tide_oracle.c follows the stock pipeline (pack every rank into a fp32
rank-major buffer, then loop over ranks), this module writes the result
straight from its definition, one (param, rank) chunk at a time, with no
packed buffer:

  out[r*Ns + off_i + e] = s * fl32(sum_{k=0..W-1} fp32(g_{k,i}[r*c_i + e]))  for r*c_i + e < numel_i
  out[...]              = +0.0                                               otherwise

  param_i[r*c_i + e]    = ag[r, off_i + e]                                   for r*c_i + e < numel_i
  param_i[...]          = +0                                                 otherwise

with S_i = ceil(d0_i / W), c_i = S_i * inner_i, off_i = sum_{j<i} c_j
(the readings are listed in tide_oracle.c).  numpy float32 adds are IEEE
round-to-nearest-even, one add per rank in rank order, so both oracles must
agree bit for bit.
"""
from __future__ import annotations

import numpy as np


def layout(world: int, shapes) -> tuple:
    """(S, c, off, Ns) for a group of parameter shapes over `world` ranks."""
    S, c, off = [], [], []
    acc = 0
    for shp in shapes:
        d0 = shp[0]
        inner = int(np.prod(shp[1:], dtype=np.int64)) if len(shp) > 1 else 1
        s = -(-d0 // world)
        S.append(s)
        c.append(s * inner)
        off.append(acc)
        acc += s * inner
    return S, c, off, acc


def _f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _numel(shp) -> int:
    return int(np.prod(shp, dtype=np.int64))


def rs_direct(world: int, shapes, grads, scale_mode: int) -> np.ndarray:
    """grads[k][i]: flat uint16 bf16 bits.  Returns fp32 [W * Ns]."""
    S, c, off, Ns = layout(world, shapes)
    out = np.zeros(world * Ns, dtype=np.float32)
    inv = np.float32(1.0) / np.float32(world)
    for i, shp in enumerate(shapes):
        n_i = _numel(shp)
        for r in range(world):
            lo = r * c[i]
            hi = min(lo + c[i], n_i)
            if hi <= lo:
                continue
            acc = _f32(grads[0][i][lo:hi])
            for k in range(1, world):
                acc = acc + _f32(grads[k][i][lo:hi])
            if scale_mode == 1:
                acc = acc * inv
            out[r * Ns + off[i]: r * Ns + off[i] + (hi - lo)] = acc
    return out


def rs_direct_f32(world: int, shapes, grads, scale_mode: int) -> np.ndarray:
    """rs_direct for fp32 gradients (grads[k][i]: flat float32, or their uint32 bits): the
    same definition with the fp32 values taken as they are."""
    S, c, off, Ns = layout(world, shapes)
    out = np.zeros(world * Ns, dtype=np.float32)
    inv = np.float32(1.0) / np.float32(world)
    g = [[np.ascontiguousarray(x).reshape(-1).view(np.float32) for x in row] for row in grads]
    for i, shp in enumerate(shapes):
        n_i = _numel(shp)
        for r in range(world):
            lo = r * c[i]
            hi = min(lo + c[i], n_i)
            if hi <= lo:
                continue
            acc = g[0][i][lo:hi].copy()
            for k in range(1, world):
                acc = acc + g[k][i][lo:hi]
            if scale_mode == 1:
                acc = acc * inv
            out[r * Ns + off[i]: r * Ns + off[i] + (hi - lo)] = acc
    return out


def ag_direct(world: int, shapes, ag: np.ndarray) -> list:
    """ag: uint16 [W, Ns].  Returns per-param padded storage (flat uint16, W*c_i each)."""
    S, c, off, Ns = layout(world, shapes)
    ag = ag.reshape(world, Ns)
    out = []
    for i, shp in enumerate(shapes):
        n_i = _numel(shp)
        p = np.zeros(world * c[i], dtype=np.uint16)
        for r in range(world):
            lo = r * c[i]
            n = max(0, min(lo + c[i], n_i) - lo)
            p[lo:lo + n] = ag[r, off[i]:off[i] + n]
        out.append(p)
    return out


def tree_sum(vals: list) -> np.ndarray:
    """Pairwise sum over a list of fp32 arrays: adjacent pairs level by level, an odd
    last element carried to the next level.  Used only to show the tree order
    stays within its error bound; the check itself compares with exact fp64 sums.
    """
    level = list(vals)
    while len(level) > 1:
        nxt = [level[j] + level[j + 1] for j in range(0, len(level) - 1, 2)]
        if len(level) % 2:
            nxt.append(level[-1])
        level = nxt
    return level[0]
