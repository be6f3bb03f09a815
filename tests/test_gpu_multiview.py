"""The multi-view preprocess (gs_preprocess_multiview) and MultiViewRenderer:
every view's records bit-exact with the oracle's single-view preprocess,
images bit-exact with the oracle's forward, argument checks; the multi-view
backward (gs_preprocess_bwd_multiview) within the suite's gradient tolerance
of the sum of the oracle's per-view gradients."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, MultiViewRenderer
from tests.gpu_helpers import assert_bits, grad_tol_check

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


NAMES = ["means", "log_scales", "quats", "opacity_logits", "sh"]


@pytest.mark.parametrize("sh_degree", [0, 1, 2, 3])
def test_multiview_backward_is_the_sum_of_the_views(sh_degree):
    # views of different sizes; the reference is the sum over views of the
    # oracle's float64 gradients, with the magnitude sums summed likewise
    sc = _mixed_size_scene(sh_degree, 160 + sh_degree)
    sc.quats[:, ::37] = 0.0  # a zero quaternion culls in every view: rows no view sees
    params = GaussianParams.from_scene(sc)
    mv = MultiViewRenderer(sc.N, sc.sh_degree, sc.cameras, capacity=64 * sc.N)
    mv.forward(params, sc.bg)
    grads = mv.backward([torch.from_numpy(sc.grad_image(p)).cuda() for p in range(len(sc.cameras))])
    torch.cuda.synchronize()
    ref_sum = {n: 0.0 for n in NAMES}
    mag_sum = {n: 0.0 for n in NAMES}
    seen = np.zeros(sc.N, bool)
    for pose, cam in enumerate(sc.cameras):
        ref = oracle.render(sc, pose)
        ob = oracle.backward(sc, cam, ref["rec"], ref["bins"], sc.grad_image(pose))
        for n in NAMES:
            ref_sum[n] = ref_sum[n] + ob["d_" + n]
            mag_sum[n] = mag_sum[n] + ob["m_" + n]
        seen |= ref["rec"]["tiles"] > 0
    assert seen.any() and not seen.all()
    for n in NAMES:
        got = grads[n].cpu().numpy()
        grad_tol_check(got, ref_sum[n], mag_sum[n], what=f"{n} summed over views")
        assert not got[..., ~seen].any(), f"{n}: a Gaussian no view sees has a gradient"


def test_multiview_backward_argument_checks():
    sc = S.random_scene(200, 64, 48, sh_degree=1, seed=170, n_poses=2)
    params = GaussianParams.from_scene(sc)
    mv = MultiViewRenderer(sc.N, sc.sh_degree, sc.cameras)
    mv.forward(params, sc.bg)
    g = [torch.zeros((3, c.height, c.width), dtype=torch.float32, device="cuda") for c in sc.cameras]
    with pytest.raises(ValueError):
        mv.backward(g[:1])
    a = mv.grads
    projs = [R._proj for R in mv.views]
    g2 = [R.grad2d for R in mv.views]
    call = lambda cams, recs, g2d: gs.gs_preprocess_bwd_multiview(
        params.means, params.log_scales, params.quats, params.opacity_logits, params.sh, params.sh_degree, sc.N,
        cams, recs, g2d, a["means"], a["log_scales"], a["quats"], a["opacity_logits"], a["sh"])
    with pytest.raises(gs.GsError):
        call([], [], [])  # no view
    with pytest.raises(gs.GsError):
        call(mv.cams * 9, projs * 9, g2 * 9)  # more than GS_MAX_VIEWS
    call(mv.cams, projs, g2)
    torch.cuda.synchronize()
