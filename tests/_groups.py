"""Small parameter groups for CPU and GPU parity tests (shapes only)."""
import numpy as np

from synth import configs


def random_group(rng: np.random.Generator, world: int, n_params: int, max_rows: int = 300,
                 max_inner: int = 70, name: str = "random") -> configs.Group:
    shapes = []
    for _ in range(n_params):
        nd = int(rng.integers(1, 4))
        d0 = int(rng.integers(0, max_rows + 1))
        if nd == 1:
            shapes.append((d0,))
        elif nd == 2:
            shapes.append((d0, int(rng.integers(1, max_inner + 1))))
        else:
            shapes.append((d0, int(rng.integers(1, 9)), int(rng.integers(1, 9))))
    return configs.Group(name, world, tuple(shapes))


def mini_sweep(world: int) -> configs.Group:
    """The sweep's structure (16 params of (64W) x cols) at a CPU-friendly size."""
    return configs.Group(f"mini_sweep_w{world}", world, tuple((64 * world, 24) for _ in range(16)))


def mini_wan() -> configs.Group:
    """Wan2.2 block structure (weights, biases, norms, a 6-row modulation) shrunk 40x in width."""
    d, f = 128, 344
    items = []
    for _ in range(2):
        for _ in range(4):
            items += [(d, d), (d,)]
        items += [(d,), (d,)]
    items += [(d,), (d,), (f, d), (f,), (d, f), (d,), (6, d)]
    return configs.Group("mini_wan", 16, tuple(items))


def degenerate() -> configs.Group:
    """Empty params, zero inner size, single rows, rows < W, an exact multiple of W."""
    return configs.Group("degenerate", 8, ((0,), (0, 5), (5, 0), (1,), (3, 7), (8, 2), (9,), (17, 3)))
