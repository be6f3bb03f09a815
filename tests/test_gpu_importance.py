"""The importance pass (gs_rasterize_fwd_importance) against the oracle.

Per Gaussian the GPU adds the same fp32 blend weights alpha*T as the oracle
(bit-exact: same alpha, same T), in fp32 through a tree: the two pixels of a
lane, a 5-level warp butterfly over the 8x8 block, then one global atomic per
(8x8 block, view), i.e. at most 4 per tile and view. All terms are positive,
so each addition's rounding error is at most 2^-24 of the final sum, and a
term passes through at most 6 + 4 * tiles * views additions:
|gpu - ref| <= (6 + 4 * tiles * views) * 2^-24 * ref; the test allows twice that.
The image outputs must equal the plain forward's bit for bit."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, Rasterizer
from tests.gpu_helpers import assert_bits, fwd_numpy

pytestmark = pytest.mark.gpu


def _check(got, ref, tiles_views):
    bound = (6.0 + 4.0 * tiles_views) * 2.0 ** -23 * ref + 1e-30
    bad = np.abs(got.astype(np.float64) - ref) > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside; worst at {np.argmax(np.abs(got - ref) / bound)}: "
                           f"got {got[bad][:3]} ref {ref[bad][:3]}")


def _gpu_importance(sc, poses, capacity=None):
    cam = sc.cameras[poses[0]]
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height, capacity=capacity)
    params = GaussianParams.from_scene(sc)
    imp = torch.zeros(sc.N, dtype=torch.float32, device="cuda")
    outs = []
    for p in poses:
        R.forward_importance(params, sc.cameras[p], imp, sc.bg, sc.lod_dist, sc.importance_q)
        torch.cuda.synchronize()
        outs.append(fwd_numpy(R))
    return imp.cpu().numpy(), outs, R


def _oracle_importance(sc, poses):
    ref = np.zeros(sc.N)
    tiles = np.zeros(sc.N)
    fwds = []
    for p in poses:
        r = oracle.render(sc, p)
        oracle.importance(r["rec"], r["bins"], sc.cameras[p], sc.N, out=ref)
        act = r["rec"]["active_idx"]
        t = r["rec"]["tiles"].astype(np.float64)
        if act is None:
            tiles += t
        else:
            tiles[act] += t[:act.size]
        fwds.append(r["fwd"])
    return ref, tiles, fwds


@pytest.mark.parametrize("name", ["sh1_ragged", "sh3_large", "culled", "config0"])
def test_importance_matches_oracle_and_image_unchanged(name):
    sc = {"sh1_ragged": lambda: S.random_scene(700, 150, 77, sh_degree=1, seed=71),
          "sh3_large": lambda: S.random_scene(2000, 200, 120, sh_degree=3, seed=72, log_scale=(-2.2, 0.5)),
          "culled": lambda: S.random_scene(1500, 128, 96, sh_degree=0, seed=73, with_importance=True,
                                           lod_dist=3.05, importance_q=0.35),
          "config0": lambda: S.make_config(0)}[name]()
    got, outs, _ = _gpu_importance(sc, [0], capacity=64 * sc.N)
    ref, tiles, fwds = _oracle_importance(sc, [0])
    assert ref.sum() > 1.0
    _check(got, ref, tiles)
    for k in ("image", "final_T", "n_contrib", "last"):
        assert_bits(outs[0][k], fwds[0][k], k)


def test_importance_sums_over_views():
    sc = S.random_scene(1200, 96, 80, sh_degree=2, seed=74, n_poses=3)
    got, _, _ = _gpu_importance(sc, [0, 1, 2], capacity=64 * sc.N)
    ref, tiles, _ = _oracle_importance(sc, [0, 1, 2])
    _check(got, ref, tiles)


def test_importance_config1():
    sc = S.make_config(1)
    got, outs, _ = _gpu_importance(sc, [0])
    ref, tiles, fwds = _oracle_importance(sc, [0])
    _check(got, ref, tiles)
    assert_bits(outs[0]["n_contrib"], fwds[0]["n_contrib"], "n_contrib")


def test_importance_feeds_the_cull():
    # the weights of an importance pass over all views are the cull's input:
    # the GPU cull on them equals the oracle's cull on the same weights
    sc = S.random_scene(3000, 128, 96, sh_degree=0, seed=75, n_poses=2, log_scale=(-2.5, 0.5))
    got, _, R = _gpu_importance(sc, [0, 1], capacity=64 * sc.N)
    sc.importance = got.astype(np.float32)
    sc.importance_q = 0.5
    cam = sc.cameras[0]
    params = GaussianParams.from_scene(sc)
    c = gs.camera(cam)
    R.cull(params, c, 0.0, sc.importance_q)
    torch.cuda.synchronize()
    cl = oracle.cull(sc, cam)
    assert_bits(R.mask.cpu().numpy(), cl["mask"], "mask")
    na = cl["n_active"]
    assert int(R.n_active.item()) == na
    assert_bits(R.active_idx[:na].cpu().numpy(), cl["active_idx"], "active_idx")
    assert 0 < na < sc.N


def test_grad2d_norm_statistic_matches_oracle():
    # on the GPU's own 2-D gradients (the same input for both), over 3 views
    # with a cull; fp32 sqrt(fma(x, x, y*y)) against float64 hypot: within
    # 2 ulp per view plus the fp32 sums over views
    sc = S.random_scene(2500, 96, 80, sh_degree=1, seed=76, n_poses=3, with_importance=True, lod_dist=3.2,
                        importance_q=0.2)
    cam = sc.cameras[0]
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height, capacity=64 * sc.N)
    params = GaussianParams.from_scene(sc)
    nsum = torch.zeros(sc.N, dtype=torch.float32, device="cuda")
    cnt = torch.zeros(sc.N, dtype=torch.int32, device="cuda")
    ref_s, ref_c = np.zeros(sc.N), np.zeros(sc.N, np.int64)
    for p in range(3):
        R.forward(params, sc.cameras[p], sc.bg, sc.lod_dist, sc.importance_q)
        R.backward(torch.from_numpy(sc.grad_image(p)).cuda())
        R.accumulate_grad_stats(nsum, cnt)
        torch.cuda.synchronize()
        na = int(R.n_active.item())
        oracle.grad2d_norm(R.grad2d.cpu().numpy()[:na], R.rec["tiles"].cpu().numpy()[:na],
                           R.active_idx.cpu().numpy()[:na], sc.N, ref_s, ref_c)
    got_s, got_c = nsum.cpu().numpy().astype(np.float64), cnt.cpu().numpy()
    np.testing.assert_array_equal(got_c, ref_c)
    assert ref_c.max() == 3 and (ref_c == 0).any()
    np.testing.assert_allclose(got_s, ref_s, rtol=4 * 2.0 ** -23, atol=0)
