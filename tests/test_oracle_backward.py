"""Pins for the oracle's backward pass.

References: float64 central finite differences of the frozen-decision forward
(every discrete decision of the fp32 run held fixed: visibility, tile lists,
skips, the 0.99 clamp, colour clamps and the stop point), and hand-derived
scalar calculus for one Gaussian over one pixel.
"""

import math

import numpy as np
import pytest

from differentiable_tile_rasterizer_b200 import synthetic as S
from tests._helpers import make_scene, params64, simple_camera

NAMES = ["means", "log_scales", "quats", "opacity_logits", "sh"]


def _fd_check(orc, sc, n_params=None, seed=0):
    cam = sc.cameras[0]
    r = orc.render(sc)
    rec, bins = r["rec"], r["bins"]
    g = sc.grad_image(0)
    an = orc.backward(sc, cam, rec, bins, g, records2d="fp64")
    base = params64(sc)
    idx = [(a, k) for a in range(5) for k in range(base[a].size)]
    if n_params is not None:
        sel = np.random.default_rng(seed).choice(len(idx), n_params, replace=False)
        idx = [idx[s] for s in sel]
    worst = 0.0
    for a, k in idx:
        p = [x.copy() for x in base]
        th = p[a].reshape(-1)[k]
        h = 1e-6 * max(1.0, abs(th))
        p[a].reshape(-1)[k] = th + h
        lp = orc.loss_frozen(p, sc, cam, rec, bins, g)
        p[a].reshape(-1)[k] = th - h
        lm = orc.loss_frozen(p, sc, cam, rec, bins, g)
        fd = (lp - lm) / (2 * h)
        ga = an["d_" + NAMES[a]].reshape(-1)[k]
        mag = an["m_" + NAMES[a]].reshape(-1)[k]
        err = abs(fd - ga) / (1e-6 * (abs(ga) + mag) + 1e-8)
        worst = max(worst, err)
        assert err <= 1.0, (NAMES[a], k, fd, ga, mag)
    return worst


def test_fd_small_sh3_all_parameters(orc):
    sc = S.random_scene(24, 40, 32, sh_degree=3, seed=21, bg=(0.2, 0.1, 0.4))
    _fd_check(orc, sc)


def test_fd_tiny_config_sampled(orc):
    _fd_check(orc, S.make_config(0), n_params=600, seed=1)


def test_fd_off_axis_rotated_camera(orc):
    sc = S.random_scene(30, 48, 40, sh_degree=2, seed=22, n_poses=3)
    sc.cameras = [sc.cameras[2]]
    _fd_check(orc, sc)


def test_fd_with_clamped_alpha_and_colour(orc):
    sc = S.random_scene(30, 40, 40, sh_degree=1, seed=23)
    sc.opacity_logits[:10] = 8.0      # alpha clamps at 0.99 near the centre
    sc.sh[0:3, 10:20] = -5.0           # colour clamps at 0
    r = orc.render(sc)
    assert (r["rec"]["rgb"][10:20, :3] == 0).any()
    _fd_check(orc, sc)


def test_single_gaussian_single_pixel_by_hand(orc):
    cam = simple_camera(1, 1, 3.0, cx=0.3, cy=0.7)
    k0 = np.array([0.8, -0.4, 1.3])
    sc = make_scene([[0.02], [-0.03], [1.5]], [[-1.0], [-1.3], [-0.8]], [[0.9], [0.2], [-0.3], [0.1]],
                    [0.7], k0.reshape(3, 1), 0, [cam], bg=(0.25, 0.5, 0.125))
    r = orc.render(sc)
    assert r["fwd"]["n_contrib"][0, 0] == 1
    g = np.array([0.3, -1.1, 0.6], np.float32)
    an = orc.backward(sc, cam, r["rec"], r["bins"], g.reshape(3, 1, 1), records2d="fp64")
    out, vis, _ = orc.project_f64(params64(sc), 0, 1, cam)
    px, py, _, o, A, B, C, cr, cg, cb = out[0]
    dx, dy = px - 0.5, py - 0.5
    p = -0.5 * (A * dx * dx + C * dy * dy) - B * dx * dy
    e = math.exp(p)
    al = o * e
    c = np.array([cr, cg, cb])
    bg = sc.bg.astype(np.float64)
    gg = g.astype(np.float64)
    # image = al c + (1 - al) bg
    dal = float(gg @ (c - bg))
    want = [dal * al * -(A * dx + B * dy), dal * al * -(B * dx + C * dy),
            dal * al * -0.5 * dx * dx, dal * al * -dx * dy, dal * al * -0.5 * dy * dy,
            dal * e, gg[0] * al, gg[1] * al, gg[2] * al]
    np.testing.assert_allclose(an["g2d"][0], want, rtol=1e-12, atol=1e-15)
    # logit: do/dlogit = o (1 - o); SH DC: colour = C0 k0 + 0.5
    assert an["d_opacity_logits"][0] == pytest.approx(dal * e * o * (1 - o), rel=1e-12)
    np.testing.assert_allclose(an["d_sh"][:, 0], gg * al * 0.28209479177387814, rtol=1e-12)


def test_magnitudes_bound_gradients_and_inactive_are_zero(orc):
    sc = S.random_scene(200, 64, 48, sh_degree=3, seed=24)
    sc.means[2, :20] = -10.0  # behind the camera
    cam = sc.cameras[0]
    r = orc.render(sc)
    an = orc.backward(sc, cam, r["rec"], r["bins"], sc.grad_image(0))
    for n in NAMES:
        assert np.all(np.abs(an["d_" + n]) <= an["m_" + n] * (1 + 1e-9) + 1e-300), n
    invisible = r["rec"]["tiles"] == 0
    assert invisible[:20].all()
    for n in NAMES:
        assert not an["d_" + n][..., invisible].any()


def test_record_point_and_fp64_point_agree_when_well_conditioned(orc):
    # the two evaluation points differ only by fp32 rounding of the records
    sc = S.random_scene(200, 64, 48, sh_degree=2, seed=25)
    cam = sc.cameras[0]
    r = orc.render(sc)
    g = sc.grad_image(0)
    a = orc.backward(sc, cam, r["rec"], r["bins"], g, records2d="fp32")
    b = orc.backward(sc, cam, r["rec"], r["bins"], g, records2d="fp64")
    assert np.all(np.abs(a["g2d"] - b["g2d"]) <= 1e-3 * np.abs(b["g2d"]) + 1e-4 * b["s2d"])
    assert np.all(a["s2d"] >= np.abs(a["g2d"]) * (1 - 1e-12))
