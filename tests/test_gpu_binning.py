"""gs_bin_sort gives the oracle's keys, values, ranges and record-order
offsets bit for bit on ragged and degenerate tile grids (one pixel, one
tile, a 300 x 7 strip, ragged edges), with big splats that span many tiles,
with a few screen-filling Gaussians in front of many small ones, and with an
instance capacity far above the count (most radix-sort CTAs past the keys)."""

import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, Rasterizer
from tests.gpu_helpers import assert_bits

pytestmark = pytest.mark.gpu

CASES = {
    "one_pixel": dict(n=50, W=1, H=1, ls=(-2.0, 0.5)),
    "one_tile": dict(n=400, W=16, H=16, ls=(-2.0, 1.0)),
    "strip_300x7": dict(n=2000, W=300, H=7, ls=(-2.0, 0.8)),
    "ragged_97x71": dict(n=3000, W=97, H=71, ls=(-2.5, 0.7)),
    "big_splats_640x480": dict(n=5000, W=640, H=480, ls=(-1.2, 0.6)),
    "many_small_800x600": dict(n=60000, W=800, H=600, ls=(-4.0, 0.6)),
}


def _check(sc, capacity, pose=0):
    cam = sc.cameras[pose]
    ref = oracle.bin_sort(oracle.preprocess(sc, cam), cam)
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height, capacity=capacity)
    R.want_offsets = True
    params = GaussianParams.from_scene(sc)
    c = gs.camera(cam)
    R.preprocess(params, c)
    R.bin_sort(c)
    torch.cuda.synchronize()
    got = R.bins_numpy()
    assert got["n_instances"] == ref["n_instances"]
    for k in ("offsets", "keys", "vals", "ranges"):
        assert_bits(got[k], ref[k], k)
    return ref["n_instances"]


@pytest.mark.parametrize("name", list(CASES))
def test_bin_sort_matches_oracle(name):
    c = CASES[name]
    sc = S.random_scene(c["n"], c["W"], c["H"], sh_degree=0, seed=300 + len(name), log_scale=c["ls"])
    I = _check(sc, None)
    _check(sc, 40 * max(I, 1024))


def test_bin_sort_screen_filling_in_front_of_small_ones():
    sc = S.random_scene(20000, 512, 384, sh_degree=0, seed=77, log_scale=(-3.5, 0.5))
    sc.log_scales[:, :5] = 1.5
    sc.means[:, :5] = 0.0
    assert _check(sc, None) > 5 * 32 * 24
