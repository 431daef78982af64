"""TIDE layout-aware FSDP2 collectives, single-GPU hot path for B200 (sm_100a).

The work is done by libtide.so (C ABI in include/tide.h); this package holds
its CUDA sources (csrc/), the build step (build.py) and a ctypes binding
(tide.py).
"""
from .tide import (  # noqa: F401
    K_AG, K_RS, K_RS_TMA, K_RS_V32, K_SLOT_RS, K_SLOT_RS_TMA, K_SLOT_RS_V32, K_STAGE, KERNEL_NAMES, TIDE_ENGINE_CE, TIDE_ENGINE_SM, TIDE_MAX_WORLD,
    TIDE_ORDER_RANK, TIDE_ORDER_TREE, TIDE_PLAN_HOST_ONLY, TIDE_PLAN_TMA, TIDE_SCALE_INV_WORLD, TIDE_SCALE_NONE,
    TIDE_TILE_ELEMS, Plan, TideError, lib,
)
