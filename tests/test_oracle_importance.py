"""Pins for the oracle's importance weights: the cross-view visibility weight
of the BlitzGS write-up (section 2.2), read as the sum over a view's pixels
of each blend's weight alpha*T.

References that are not the oracle's own walk: the telescoping identity
sum_k alpha_k T_k = 1 - T_final per pixel (with the fp32 rounding bound of
the T recursion), float64 closed forms for one Gaussian and for two stacked
Gaussians, and the sub-scene of the active Gaussians for culled views."""

import numpy as np

import oracle
from differentiable_tile_rasterizer_b200 import synthetic as S
from tests._helpers import make_scene, simple_camera

EPS = 2.0 ** -24
AMIN = np.float32(1.0 / 255.0)


def _view(sc, pose=0):
    r = oracle.render(sc, pose)
    imp = oracle.importance(r["rec"], r["bins"], sc.cameras[pose], sc.N)
    return r, imp


def test_weights_sum_to_covered_fraction():
    # per pixel sum_k fl(alpha_k T_k) + T_final = 1 up to 2 roundings per
    # T update and one per weight: |error| <= (2 n + 1) eps
    for sc in (S.random_scene(300, 70, 45, sh_degree=1, seed=61),
               S.random_scene(800, 128, 96, sh_degree=0, seed=62, log_scale=(-2.0, 0.5)),
               S.make_config(0)):
        r, imp = _view(sc)
        T = r["fwd"]["final_T"].astype(np.float64)
        nblend = int(r["fwd"]["n_contrib"].sum())
        covered = float((1.0 - T).sum())
        assert nblend > 0 and covered > 0.1
        assert abs(imp.sum() - covered) <= (2 * nblend + T.size) * EPS
        assert np.all(imp >= 0)
        # Gaussians that reach no tile get no weight
        assert not imp[r["rec"]["tiles"] == 0].any()


def _alpha64(rec, i, xs, ys):
    """Float64 alpha of record i at pixel centres (xs, ys), and the pixels
    whose alpha lies within 1e-5 of the 1/255 threshold (either side may
    decide those)."""
    px, py, _, o = rec["xyzo"][i].astype(np.float64)
    A, B, C, _ = rec["conic"][i].astype(np.float64)
    dx, dy = px - xs, py - ys
    p = -0.5 * (A * dx * dx + C * dy * dy) - B * dx * dy
    a = np.minimum(0.99, o * np.exp(p))
    return a, np.abs(a - float(AMIN)) < 1e-5


def _in_rect(rec, i, us, vs):
    x0, y0, x1, y1 = rec["rect"][i].astype(np.int64)
    return (us // 16 >= x0) & (us // 16 < x1) & (vs // 16 >= y0) & (vs // 16 < y1)


def _grid(cam):
    vs, us = np.mgrid[0:cam.height, 0:cam.width]
    return us.ravel(), vs.ravel(), us.ravel() + 0.5, vs.ravel() + 0.5


def test_single_gaussian_is_its_sum_of_alpha():
    cam = simple_camera(80, 64, 60.0, cx=37.3, cy=30.9)
    sc = make_scene([[0.05], [-0.02], [2.0]], [[-1.6], [-2.1], [-1.9]], [[0.9], [0.3], [-0.2], [0.1]],
                    [1.2], np.full((3, 1), 0.4), 0, [cam])
    r, imp = _view(sc)
    us, vs, xs, ys = _grid(cam)
    a, amb = _alpha64(r["rec"], 0, xs, ys)
    keep = _in_rect(r["rec"], 0, us, vs) & (a >= float(AMIN))
    ref = a[keep].sum()
    n_amb = int((amb & _in_rect(r["rec"], 0, us, vs)).sum())
    assert ref > 1.0
    assert abs(imp[0] - ref) <= 1e-5 * ref + n_amb * float(AMIN)


def test_two_stacked_gaussians_attribution_and_occlusion():
    cam = simple_camera(64, 64, 64.0, cx=31.7, cy=32.4)
    means = [[0.0, 0.0], [0.0, 0.0], [1.5, 3.0]]  # same axis, the first in front
    ls = [[-1.8, -1.2], [-1.8, -1.2], [-1.8, -1.2]]
    q = [[1.0, 1.0], [0.0, 0.0], [0.0, 0.0], [0.0, 0.0]]
    sc = make_scene(means, ls, q, [0.4, 2.0], np.full((3, 2), 0.3), 0, [cam])
    r, imp = _view(sc)
    rec = r["rec"]
    us, vs, xs, ys = _grid(cam)
    a0, amb0 = _alpha64(rec, 0, xs, ys)
    a1, amb1 = _alpha64(rec, 1, xs, ys)
    in0, in1 = _in_rect(rec, 0, us, vs), _in_rect(rec, 1, us, vs)
    b0 = in0 & (a0 >= float(AMIN))
    b1 = in1 & (a1 >= float(AMIN))
    ref0 = a0[b0].sum()
    ref1 = (a1 * np.where(b0, 1.0 - a0, 1.0))[b1].sum()  # behind the first
    n_amb = int(((amb0 & in0) | (amb1 & in1)).sum())
    assert ref0 > 1.0 and ref1 > 1.0
    assert abs(imp[0] - ref0) <= 1e-5 * ref0 + n_amb * float(AMIN)
    assert abs(imp[1] - ref1) <= 1e-5 * ref1 + n_amb * float(AMIN)
    # the same two Gaussians given in the other index order swap their weights
    sw = make_scene(np.asarray(means)[:, ::-1], np.asarray(ls)[:, ::-1], np.asarray(q)[:, ::-1],
                    [2.0, 0.4], np.full((3, 2), 0.3), 0, [cam])
    _, imp_sw = _view(sw)
    np.testing.assert_allclose(imp_sw, imp[::-1], rtol=1e-12, atol=0)  # (fp64 sums, any order)


def test_culled_view_maps_records_to_gaussians():
    sc = S.random_scene(600, 96, 64, sh_degree=0, seed=63, with_importance=True, lod_dist=3.05,
                        importance_q=0.4)
    r, imp = _view(sc)
    act = r["rec"]["active_idx"]
    assert 0 < act.size < sc.N
    # the same view rendered from the active Gaussians alone, without a cull
    sub = S.Scene("sub", act.size, sc.sh_degree, sc.means[:, act], sc.log_scales[:, act], sc.quats[:, act],
                  sc.opacity_logits[act], sc.sh[:, act], sc.cameras, sc.bg, True)
    _, imp_sub = _view(sub)
    np.testing.assert_allclose(imp[act], imp_sub, rtol=1e-12, atol=0)
    culled = np.ones(sc.N, bool)
    culled[act] = False
    assert not imp[culled].any()


def test_views_add_up():
    sc = S.random_scene(400, 64, 48, sh_degree=1, seed=64, n_poses=3)
    total = np.zeros(sc.N)
    parts = []
    for p in range(3):
        r = oracle.render(sc, p)
        parts.append(oracle.importance(r["rec"], r["bins"], sc.cameras[p], sc.N))
        oracle.importance(r["rec"], r["bins"], sc.cameras[p], sc.N, out=total)
    np.testing.assert_allclose(total, parts[0] + parts[1] + parts[2], rtol=1e-12, atol=0)


def test_grad2d_norm_statistic_is_the_plain_definition():
    # the densification statistic: per visible record, hypot(dpx, dpy) added
    # to its Gaussian, one view counted; checked element by element with
    # math.hypot over a permuted active list with invisible records
    import math
    rng = np.random.default_rng(65)
    n, N = 50, 80
    g2 = rng.normal(0, 1, (n, 12)).astype(np.float32)
    tiles = rng.integers(-1, 3, n).astype(np.int32)
    act = rng.permutation(N)[:n].astype(np.int32)
    s, c = oracle.grad2d_norm(g2, tiles, act, N)
    s2, c2 = oracle.grad2d_norm(g2, tiles, act, N, s.copy(), c.copy())
    ref_s, ref_c = np.zeros(N), np.zeros(N, np.int64)
    for i in range(n):
        if tiles[i] > 0:
            ref_s[act[i]] += math.hypot(float(g2[i, 0]), float(g2[i, 1]))
            ref_c[act[i]] += 1
    np.testing.assert_allclose(s, ref_s, rtol=1e-15, atol=0)
    np.testing.assert_array_equal(c, ref_c)
    np.testing.assert_allclose(s2, 2 * ref_s, rtol=1e-15, atol=0)
    np.testing.assert_array_equal(c2, 2 * ref_c)
