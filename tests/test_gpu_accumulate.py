"""gs_preprocess_bwd_accumulate: the parameter gradient of a loss summed over
views, added view by view. Exactly the fp32 sum of the views' overwritten
gradients (gs_preprocess_bwd) taken in the same order, within the suite's
tolerance of the sum of the oracle's per-view gradients, and it leaves the
rows of Gaussians no view sees untouched."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, Rasterizer
from tests.gpu_helpers import grad_tol_check

pytestmark = pytest.mark.gpu

NAMES = ["means", "log_scales", "quats", "opacity_logits", "sh"]


@pytest.mark.parametrize("cull", [False, True])
def test_accumulated_views_equal_the_sum_of_views(cull):
    sc = S.random_scene(4000, 160, 120, sh_degree=3, seed=150, n_poses=3, log_scale=(-2.5, 0.6),
                        with_importance=cull, lod_dist=3.4 if cull else 0.0, importance_q=0.3 if cull else 0.0)
    params = GaussianParams.from_scene(sc)
    cam0 = sc.cameras[0]
    R = Rasterizer(sc.N, sc.sh_degree, cam0.width, cam0.height)
    acc = {n: torch.zeros_like(R.grads[n]) for n in NAMES}
    seen = np.zeros(sc.N, bool)
    per_view = []
    ref_sum = {n: 0.0 for n in NAMES}
    mag_sum = {n: 0.0 for n in NAMES}
    for pose in range(len(sc.cameras)):
        cam = sc.cameras[pose]
        g = torch.from_numpy(sc.grad_image(pose)).cuda()
        R.forward(params, cam, sc.bg, sc.lod_dist, sc.importance_q)
        R.backward(g, accumulate_into=acc)
        # the view's own (overwritten) gradients from the same 2-D gradients:
        # those are float atomic sums in unspecified order, so two backward
        # runs need not agree bit for bit, but one set of them must
        act = R.active_idx if R.culled else None
        na = R.n_active if R.culled else None
        mask = R.mask if R.culled else None
        gg = R.grads
        gs.gs_preprocess_bwd(params.means, params.log_scales, params.quats, params.opacity_logits, params.sh,
                             params.sh_degree, R.N, act, na, mask, R.cam, R._proj, R.grad2d, gg["means"],
                             gg["log_scales"], gg["quats"], gg["opacity_logits"], gg["sh"])
        torch.cuda.synchronize()
        per_view.append({n: gg[n].cpu().numpy().copy() for n in NAMES})
        ref = oracle.render(sc, pose)
        ob = oracle.backward(sc, cam, ref["rec"], ref["bins"], sc.grad_image(pose))
        for n in NAMES:
            ref_sum[n] = ref_sum[n] + ob["d_" + n]
            mag_sum[n] = mag_sum[n] + ob["m_" + n]
        na = ref["rec"]["n_active"]
        vis = ref["rec"]["tiles"][:na] > 0
        gid = np.flatnonzero(vis) if ref["rec"]["active_idx"] is None else ref["rec"]["active_idx"][vis]
        seen[gid] = True
    for n in NAMES:
        want = per_view[0][n]
        for v in per_view[1:]:
            want = (want + v[n]).astype(np.float32)
        # exact equality of values: the zero the sum starts from turns a -0
        # term (a clamped colour's SH gradient) into +0, the only bit that
        # may differ
        got = acc[n].cpu().numpy()
        assert np.array_equal(got, want), f"{n}: {int(np.count_nonzero(got != want))} values differ"
        grad_tol_check(acc[n].cpu().numpy(), ref_sum[n], mag_sum[n], what=f"{n} summed over views")
    assert seen.any()


def test_accumulate_leaves_unseen_rows_untouched():
    sc = S.random_scene(3000, 96, 64, sh_degree=1, seed=151, log_scale=(-2.5, 0.6))
    params = GaussianParams.from_scene(sc)
    cam = sc.cameras[0]
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height)
    R.forward(params, cam, sc.bg)
    acc = {n: torch.full_like(R.grads[n], 3.25) for n in NAMES}
    R.backward(torch.from_numpy(sc.grad_image(0)).cuda(), accumulate_into=acc)
    torch.cuda.synchronize()
    invisible = (R.rec["tiles"] <= 0).cpu().numpy()
    assert invisible.any()
    for n in NAMES:
        a = acc[n].cpu().numpy()
        assert np.all(a[..., invisible] == np.float32(3.25)), n
