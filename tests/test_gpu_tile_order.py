"""The tile schedule (gs_tile_order) and the raster launches that take it.

The order is a permutation of the tiles whose floor(log2) list-length classes
do not increase along it (empty lists last). It is a schedule only: the
forward outputs with and without it are bit-identical, and so are the
backward's gradients up to the order of their fp32 atomic sums (checked
against the oracle with the suite's gradient tolerance)."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, Rasterizer
from tests.gpu_helpers import assert_bits, grad_tol_check

pytestmark = pytest.mark.gpu

NAMES = ["means", "log_scales", "quats", "opacity_logits", "sh"]


def _length_class(lens):
    lens = np.asarray(lens, dtype=np.uint64)
    out = np.zeros(lens.shape, dtype=np.int64)
    nz = lens > 0
    out[nz] = np.floor(np.log2(lens[nz].astype(np.float64))).astype(np.int64) + 1
    return out


def _check_order(order, ranges):
    r = ranges.astype(np.int64)
    lens = r[:, 1] - r[:, 0]
    TT = lens.shape[0]
    assert np.array_equal(np.sort(order), np.arange(TT)), "not a permutation"
    cls = _length_class(lens[order])
    assert np.all(np.diff(cls) <= 0), "length classes increase along the order"


def _render(sc, schedule, pose=0, backward=True):
    cam = sc.cameras[pose]
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height)
    R.schedule_tiles = schedule
    R.want_offsets = True
    p = GaussianParams.from_scene(sc)
    R.forward(p, cam, sc.bg)
    out = {k: v.cpu().numpy() for k, v in (("image", R.image), ("final_T", R.final_T),
                                           ("n_contrib", R.n_contrib), ("last", R.last))}
    if backward:
        g = R.backward(torch.from_numpy(sc.grad_image(pose)).cuda())
        out.update({"d_" + n: g[n].cpu().numpy() for n in NAMES})
    torch.cuda.synchronize()
    return R, out


@pytest.mark.parametrize("seed,W,H", [(140, 211, 133), (141, 64, 48), (142, 1000, 17)])
def test_order_is_a_length_class_sorted_permutation(seed, W, H):
    sc = S.random_scene(3000, W, H, sh_degree=1, seed=seed, log_scale=(-3.0, 0.3))
    R, _ = _render(sc, True, backward=False)
    ranges = R.ranges.cpu().numpy().view(np.uint32)
    _check_order(R.tile_order.cpu().numpy()[: R.TT].astype(np.int64), ranges)
    # the lengths span several classes, so the order is not trivial
    assert len(set(_length_class(ranges[:, 1].astype(np.int64) - ranges[:, 0]).tolist())) >= 3


def test_order_of_empty_lists_and_no_tiles():
    TT = 5000
    ranges = torch.zeros((TT, 2), dtype=torch.int32, device="cuda")
    order = torch.full((TT,), -1, dtype=torch.int32, device="cuda")
    gs.gs_tile_order(ranges, TT, order)
    assert np.array_equal(np.sort(order.cpu().numpy()), np.arange(TT))
    # one long list, the rest short: the long one comes first
    r = np.zeros((TT, 2), np.int32)
    r[:, 1] = 1
    r[1234] = (0, 1 << 20)
    gs.gs_tile_order(torch.from_numpy(r).cuda(), TT, order)
    o = order.cpu().numpy()
    assert o[0] == 1234 and np.array_equal(np.sort(o), np.arange(TT))
    gs.gs_tile_order(ranges, 0, order)  # no tiles: nothing to do
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", ["ragged", "dense"])
def test_schedule_changes_no_forward_bit_and_keeps_gradients(name):
    if name == "ragged":
        sc = S.random_scene(2500, 173, 95, sh_degree=2, seed=143, log_scale=(-2.5, 0.4))
    else:
        sc = S.random_scene(6000, 128, 128, sh_degree=3, seed=144, log_scale=(-2.0, 0.6), n_poses=2)
    for pose in range(len(sc.cameras)):
        _, a = _render(sc, True, pose)
        _, b = _render(sc, False, pose)
        for k in ("image", "final_T", "n_contrib", "last"):
            assert_bits(a[k], b[k], f"{k} pose {pose}")
        sub = S.Scene(sc.name, sc.N, sc.sh_degree, sc.means, sc.log_scales, sc.quats, sc.opacity_logits, sc.sh,
                      [sc.cameras[pose]], sc.bg, True)
        ref = oracle.render(sub)
        assert_bits(a["image"], ref["fwd"]["image"], "image vs oracle")
        ob = oracle.backward(sub, sub.cameras[0], ref["rec"], ref["bins"], sc.grad_image(pose))
        for n in NAMES:
            grad_tol_check(a["d_" + n], ob["d_" + n], ob["m_" + n], what=f"{n} scheduled pose {pose}")
            grad_tol_check(b["d_" + n], ob["d_" + n], ob["m_" + n], what=f"{n} natural pose {pose}")


def test_importance_pass_with_schedule():
    sc = S.random_scene(2000, 150, 110, sh_degree=1, seed=145)
    cam = sc.cameras[0]
    p = GaussianParams.from_scene(sc)
    imps = []
    for schedule in (True, False):
        R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height)
        R.schedule_tiles = schedule
        imp = torch.zeros(sc.N, dtype=torch.float32, device="cuda")
        R.forward_importance(p, cam, imp, sc.bg)
        imps.append((R.image.cpu().numpy(), imp.cpu().numpy()))
    assert_bits(imps[0][0], imps[1][0], "image")
    # per-(Gaussian, tile) atomic sums in another order: a few ulps apart
    np.testing.assert_allclose(imps[0][1], imps[1][1], rtol=1e-5, atol=1e-6)
