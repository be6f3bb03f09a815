"""Host-side pieces of the index-interleaved multi-GPU render (CPU): the row
bands of the ranks partition the tile rows in order, and rank r holds the
Gaussians r, r + G, r + 2G, ... of every parameter plane."""

import numpy as np
import pytest
import torch

from differentiable_tile_rasterizer_b200.multigpu import band_rows, local_params
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams


@pytest.mark.parametrize("TH,G", [(68, 8), (68, 3), (5, 8), (1, 1), (135, 7), (17, 32)])
def test_bands_partition_the_tile_rows(TH, G):
    bands = [band_rows(r, G, TH) for r in range(G)]
    assert bands[0][0] == 0 and bands[-1][1] == TH
    for (lo, hi), (lo2, _) in zip(bands, bands[1:]):
        assert lo <= hi == lo2  # contiguous, in rank order, possibly empty
    sizes = [hi - lo for lo, hi in bands]
    assert max(sizes) - min(sizes) <= 1  # as even as integers allow


@pytest.mark.parametrize("N,G", [(10, 3), (7, 7), (5, 8), (1000, 4)])
def test_local_params_interleave_by_index(N, G):
    rng = np.random.default_rng(N + G)
    t = lambda *shape: torch.from_numpy(rng.standard_normal(shape).astype(np.float32))
    p = GaussianParams(t(3, N), t(3, N), t(4, N), t(N), t(48, N), 3, t(N))
    parts = [local_params(p, r, G) for r in range(G)]
    assert sum(q.N for q in parts) == N
    for name in ("means", "log_scales", "quats", "opacity_logits", "sh", "importance"):
        full = getattr(p, name).numpy()
        back = np.zeros_like(full)
        for r, q in enumerate(parts):
            local = getattr(q, name)
            assert local.is_contiguous()
            back[..., r::G] = local.numpy()
        np.testing.assert_array_equal(back, full, err_msg=name)


def _best_max_band(cost, world):
    """Least largest band sum over every contiguous partition (brute force)."""
    import itertools
    TH = len(cost)
    best = None
    for cuts in itertools.combinations_with_replacement(range(TH + 1), world - 1):
        starts = [0, *cuts, TH]
        m = max(sum(cost[a:b]) for a, b in zip(starts, starts[1:]))
        best = m if best is None else min(best, m)
    return best


@pytest.mark.parametrize("seed", range(12))
def test_balanced_bands_reach_the_least_largest_band(seed):
    from differentiable_tile_rasterizer_b200.multigpu import balance_bands
    rng = np.random.default_rng(seed)
    TH = int(rng.integers(1, 9))
    world = int(rng.integers(1, 5))
    cost = [int(c) for c in rng.integers(0, 50, TH) * (rng.random(TH) < 0.8)]
    starts = balance_bands(cost, world)
    assert len(starts) == world + 1 and starts[0] == 0 and starts[-1] == TH
    assert all(a <= b for a, b in zip(starts, starts[1:]))
    if sum(cost) > 0:
        got = max(sum(cost[a:b]) for a, b in zip(starts, starts[1:]))
        assert got == _best_max_band(cost, world)


def test_balanced_bands_follow_the_work():
    from differentiable_tile_rasterizer_b200.multigpu import balance_bands, equal_bands
    assert balance_bands([0.0] * 68, 8) == equal_bands(8, 68)
    cost = [1.0] * 60 + [100.0] * 8  # the work sits in the last rows
    starts = balance_bands(cost, 4)
    assert starts[1] > 40 and starts[-1] == 68
    sums = [sum(cost[a:b]) for a, b in zip(starts, starts[1:])]
    assert max(sums) < 0.5 * sum(cost)
