"""The seeded input generator: published SplitMix64 outputs, determinism, statistics."""
import numpy as np
import pytest

import synth
from synth import configs


def test_splitmix64_published_outputs():
    # A SplitMix64 stream seeded with 0 yields, in order, these three outputs
    # (Vigna's reference splitmix64.c); our stateless form mixes state + k*gamma.
    gamma = 0x9E3779B97F4A7C15
    mask = (1 << 64) - 1
    assert synth.splitmix64(0) == 0xE220A8397B1DCDAF
    assert synth.splitmix64(gamma) == 0x6E789E6AA1B965F4
    assert synth.splitmix64((2 * gamma) & mask) == 0x06C45D188009454F


def test_deterministic_and_keyed():
    a = synth.fill_bf16(4096, 1, 0, 3, 2, 1e-3)
    b = synth.fill_bf16(4096, 1, 0, 3, 2, 1e-3)
    assert np.array_equal(a, b)
    for other in (synth.fill_bf16(4096, 2, 0, 3, 2, 1e-3), synth.fill_bf16(4096, 1, 1, 3, 2, 1e-3),
                  synth.fill_bf16(4096, 1, 0, 4, 2, 1e-3), synth.fill_bf16(4096, 1, 0, 3, 3, 1e-3)):
        assert np.mean(a == other) < 0.05


def test_offset_and_gather_agree():
    full = synth.fill_bf16(10000, 7, 0, 1, 5, 1e-3)
    part = synth.fill_bf16(1000, 7, 0, 1, 5, 1e-3, idx0=9000)
    assert np.array_equal(full[9000:], part)
    idx = np.array([0, 17, 9999, 4321], dtype=np.int64)
    assert np.array_equal(synth.gather_bf16(idx, 7, 0, 1, 5, 1e-3), full[idx])


@pytest.mark.parametrize("sigma", [1e-3, 0.02])
def test_distribution(sigma):
    x = synth.fill_bf16(1 << 18, 1, 0, 0, 0, sigma)
    f = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert abs(f.mean()) < 0.01 * sigma
    assert abs(f.std() / sigma - 1.0) < 0.01
    # Irwin-Hall(4): bounded support at about 3.46 sigma, no NaN/Inf, no -0.
    assert np.all(np.isfinite(f)) and np.abs(f).max() <= 3.47 * sigma
    assert not np.any(x == 0x8000)


def test_matches_recipe_in_python():
    """The C code follows the documented recipe (checked against a big-int restatement)."""
    M = (1 << 64) - 1

    def sm(v):
        z = (v + 0x9E3779B97F4A7C15) & M
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
        return z ^ (z >> 31)

    seed, stream, rank, param = 11, 1, 5, 9
    key = sm(sm(seed) ^ ((stream << 48) ^ (rank << 32) ^ param))
    mul = np.float32(synth.sigma_scale(0.02))
    got = synth.fill_bf16(64, seed, stream, rank, param, 0.02)
    for idx in range(64):
        h = sm(key ^ idx)
        s = sum((h >> (16 * L)) & 0xFFFF for L in range(4)) - 131070
        x = np.float32(s) * mul
        u = int(np.array([x], dtype=np.float32).view(np.uint32)[0])
        u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
        assert got[idx] == u


def test_zero_experts():
    g = configs.qwen3moe()
    assert g.n_zero_experts == 6
    masks = [synth.zero_experts(128, 6, 1, r) for r in range(8)]
    for m in masks:
        assert m.sum() == 6
    assert len({tuple(np.nonzero(m)[0]) for m in masks}) > 1
    assert np.array_equal(masks[3], synth.zero_experts(128, 6, 1, 3))
    zp = synth.zero_grad_params(g, 1, 0)
    assert len(zp) == 18
    assert all(7 <= i < 7 + 3 * 128 for i in zp)
