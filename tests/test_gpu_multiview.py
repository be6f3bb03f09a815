"""The multi-view preprocess (gs_preprocess_multiview) and MultiViewRenderer:
every view's records bit-exact with the oracle's single-view preprocess,
images bit-exact with the oracle's forward, argument checks."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, MultiViewRenderer
from tests.gpu_helpers import assert_bits

pytestmark = pytest.mark.gpu

REC_KEYS = ("xyzo", "conic", "rgb", "radius", "rect", "tiles")


def _mixed_size_scene(sh_degree, seed):
    sc = S.random_scene(1500, 96, 64, sh_degree=sh_degree, seed=seed, n_poses=3, log_scale=(-2.5, 0.5))
    # give the views different image sizes (ragged tile tails)
    for cam, (w, h) in zip(sc.cameras, [(96, 64), (70, 45), (129, 33)]):
        cam.cx, cam.cy = cam.cx * w / cam.width, cam.cy * h / cam.height
        cam.width, cam.height = w, h
    return sc


@pytest.mark.parametrize("sh_degree", [0, 1, 2, 3])
def test_multiview_records_bitexact(sh_degree):
    sc = _mixed_size_scene(sh_degree, 80 + sh_degree)
    mv = MultiViewRenderer(sc.N, sc.sh_degree, sc.cameras, capacity=64 * sc.N)
    mv.forward(GaussianParams.from_scene(sc), sc.bg)
    torch.cuda.synchronize()
    for v, cam in enumerate(sc.cameras):
        ref = oracle.preprocess(sc, cam)
        got = mv.views[v].records_numpy()
        for k in REC_KEYS:
            assert_bits(got[k], ref[k], f"view {v} {k}")


def test_multiview_images_bitexact():
    sc = _mixed_size_scene(3, 85)
    mv = MultiViewRenderer(sc.N, sc.sh_degree, sc.cameras, capacity=64 * sc.N)
    imgs = mv.forward(GaussianParams.from_scene(sc), sc.bg)
    torch.cuda.synchronize()
    for v, cam in enumerate(sc.cameras):
        rec = oracle.preprocess(sc, cam)
        bins = oracle.bin_sort(rec, cam)
        ref = oracle.raster_fwd(rec, bins, cam, sc.bg)
        assert_bits(imgs[v].cpu().numpy(), ref["image"], f"image {v}")
        assert_bits(mv.views[v].n_contrib.cpu().numpy(), ref["n_contrib"], f"n_contrib {v}")


def test_multiview_argument_checks():
    sc = S.random_scene(10, 32, 32, sh_degree=0, seed=86)
    p = GaussianParams.from_scene(sc)
    c = gs.camera(sc.cameras[0])
    mv = MultiViewRenderer(sc.N, 0, sc.cameras)
    outs = [mv.views[0]._proj] * (gs.GS_MAX_VIEWS + 1)
    with pytest.raises(gs.GsError):
        gs.gs_preprocess_multiview(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh, 0, sc.N,
                                   [c] * len(outs), outs)
    gs.gs_preprocess_multiview(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh, 0, sc.N, [], [])
    with pytest.raises(ValueError):
        MultiViewRenderer(sc.N, 0, [])
