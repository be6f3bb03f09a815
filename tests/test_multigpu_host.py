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
