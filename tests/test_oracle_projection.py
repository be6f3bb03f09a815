"""Pins for the oracle's per-Gaussian projection (preprocess).

Independent references: closed forms for an isotropic Gaussian on the optical
axis, scipy's quaternion-to-matrix routine with a numerically differentiated
pinhole map for Sigma' = J W Sigma W^T J^T + 0.3 I, numpy eigenvalues for the
3-sigma radius, interval overlap for the tile rect, scipy's expit for opacity
and scipy's spherical harmonics for colour.
"""

import math

import numpy as np
import pytest
from scipy.spatial.transform import Rotation
from scipy.special import expit

from differentiable_tile_rasterizer_b200 import synthetic as S
from tests._helpers import make_scene, params64, simple_camera
from tests.test_oracle_sh import _scipy_real_sh


def _iso_scene(z, s, f, W=96, H=80, logit=0.3, q=(0.3, -0.5, 0.7, 0.1)):
    cam = simple_camera(W, H, f)
    q = np.asarray(q, np.float64)
    q = q / np.linalg.norm(q)
    sc = make_scene([[0.0], [0.0], [z]], [[math.log(s)]] * 3, q.reshape(4, 1), [logit],
                    np.zeros((3, 1)), 0, [cam])
    return sc, cam


@pytest.mark.parametrize("z,s,f", [(3.0, 0.05, 60.0), (5.0, 0.3, 100.0), (1.5, 0.01, 200.0)])
def test_isotropic_closed_form(orc, z, s, f):
    sc, cam = _iso_scene(z, s, f)
    out, vis, rad = orc.project_f64(params64(sc), 0, 1, cam)
    s_eff = math.exp(np.float64(np.float32(math.log(s))))  # the stored log-scale is fp32
    sig2 = (f * s_eff / z) ** 2 + 0.3
    px, py, depth, op, A, B, C = out[0, :7]
    assert vis[0] == 1
    assert px == pytest.approx(cam.cx, abs=1e-12) and py == pytest.approx(cam.cy, abs=1e-12)
    assert depth == pytest.approx(z)
    assert A == pytest.approx(1 / sig2, rel=1e-9) and C == pytest.approx(1 / sig2, rel=1e-9)
    assert abs(B) < 1e-12 / sig2
    assert rad[0] == math.ceil(3 * math.sqrt(sig2))
    # fp32 spec mode agrees
    rec = orc.preprocess(sc, cam)
    assert rec["radius"][0] == rad[0]
    assert rec["conic"][0, 0] == pytest.approx(1 / sig2, rel=2e-6)
    assert rec["xyzo"][0, 0] == pytest.approx(cam.cx, abs=1e-5)


def test_isotropic_independent_of_rotation(orc):
    outs = []
    for seed in range(5):
        q = np.random.default_rng(seed).standard_normal(4)
        sc, cam = _iso_scene(4.0, 0.2, 80.0, q=q)
        outs.append(orc.project_f64(params64(sc), 0, 1, cam)[0][0, :7])
    outs = np.array(outs)
    assert np.abs(outs - outs[0]).max() < 1e-12


def _random_gaussians(n, seed):
    rng = np.random.default_rng(seed)
    means = rng.uniform(-1, 1, (3, n))
    log_scales = rng.normal(-2.5, 0.6, (3, n))
    quats = rng.standard_normal((4, n))
    logits = rng.normal(0, 1.5, n)
    sh = np.concatenate([rng.random((3, n)), rng.normal(0, 0.3, (45, n))])
    return [a.astype(np.float32) for a in (means, log_scales, quats, logits, sh)]


def _reference_projection(sc, cam):
    """Sigma', centre and colour from library routines (fp64)."""
    W = cam.R.astype(np.float64)
    t0 = cam.t.astype(np.float64)
    means, ls, q, lg, sh = params64(sc)
    N = sc.N
    out = []
    for g in range(N):
        mu = means[:, g]
        t = W @ mu + t0
        rot = Rotation.from_quat([q[1, g], q[2, g], q[3, g], q[0, g]]).as_matrix()
        Sig = rot @ np.diag(np.exp(2 * ls[:, g])) @ rot.T

        def proj(tt):
            return np.array([cam.fx * tt[0] / tt[2] + cam.cx, cam.fy * tt[1] / tt[2] + cam.cy])

        J = np.zeros((2, 3))
        for m in range(3):
            h = 1e-5 * max(1.0, abs(t[m]))
            e = np.zeros(3)
            e[m] = h
            J[:, m] = (proj(t + e) - proj(t - e)) / (2 * h)
        Sp = J @ W @ Sig @ W.T @ J.T + 0.3 * np.eye(2)
        lam = np.linalg.eigvalsh(Sp).max()
        d = mu - cam.campos.astype(np.float64)
        Y = _scipy_real_sh((d / np.linalg.norm(d))[None, :])[0, :sc.K]
        col = np.array([Y @ sh[ch::3, g] for ch in range(3)]) + 0.5
        out.append(dict(t=t, Sp=Sp, conic=np.linalg.inv(Sp), lam=lam, px=proj(t),
                        op=expit(lg[g]), col=col))
    return out


@pytest.mark.parametrize("sh_degree", [0, 1, 2, 3])
def test_projection_against_library_routines(orc, sh_degree):
    K = (sh_degree + 1) ** 2
    means, ls, q, lg, sh = _random_gaussians(200, 7 + sh_degree)
    cam = S.look_at((0.4, -0.3, -4.0), (0, 0, 0), (0, -1, 0), 300, 280, 160, 120, 320, 240)
    sc = make_scene(means, ls, q, lg, sh[:3 * K], sh_degree, [cam])
    ref = _reference_projection(sc, cam)
    out, vis, rad = orc.project_f64(params64(sc), sh_degree, sc.N, cam)
    rec = orc.preprocess(sc, cam)
    checked = 0
    for g in range(sc.N):
        r = ref[g]
        if not vis[g]:
            continue
        checked += 1
        A, B, C = out[g, 4:7]
        np.testing.assert_allclose([A, B, C], [r["conic"][0, 0], r["conic"][0, 1], r["conic"][1, 1]],
                                   rtol=1e-7, atol=1e-9 * abs(r["conic"][0, 0]))
        np.testing.assert_allclose(out[g, 0:2], r["px"], rtol=1e-12, atol=1e-9)
        assert out[g, 3] == pytest.approx(r["op"], rel=1e-12)
        np.testing.assert_allclose(out[g, 7:10], np.maximum(r["col"], 0), atol=1e-12)
        rr = 3 * math.sqrt(r["lam"])
        if abs(rr - round(rr)) > 1e-6:
            assert rad[g] == math.ceil(rr)
        # fp32 spec mode against the same references
        np.testing.assert_allclose(rec["conic"][g, :3], [r["conic"][0, 0], r["conic"][0, 1], r["conic"][1, 1]],
                                   rtol=2e-4, atol=2e-4 * abs(r["conic"][0, 0]))
        np.testing.assert_allclose(rec["xyzo"][g, :2], r["px"], rtol=1e-6, atol=1e-4)
        assert rec["xyzo"][g, 3] == pytest.approx(r["op"], rel=1e-6)
        np.testing.assert_allclose(rec["rgb"][g, :3], np.maximum(r["col"], 0), atol=5e-6)
    assert checked > 100


def test_rect_is_tile_overlap_of_the_3sigma_square(orc):
    sc = S.make_config(0)
    cam = sc.cameras[0]
    rec = orc.preprocess(sc, cam)
    vis = rec["tiles"] > 0
    assert vis.sum() > 200
    for g in np.nonzero(vis)[0]:
        px, py = np.float64(rec["xyzo"][g, 0]), np.float64(rec["xyzo"][g, 1])
        r = np.float64(rec["radius"][g])
        tx = [t for t in range(cam.tiles_x) if 16 * t <= px + r and px - r < 16 * (t + 1)]
        ty = [t for t in range(cam.tiles_y) if 16 * t <= py + r and py - r < 16 * (t + 1)]
        x0, y0, x1, y1 = rec["rect"][g].astype(int)
        assert (x0, x1) == (tx[0], tx[-1] + 1)
        assert (y0, y1) == (ty[0], ty[-1] + 1)
        assert rec["tiles"][g] == (x1 - x0) * (y1 - y0)


def test_culling_cases(orc):
    cam = simple_camera(64, 64, 50.0, near=0.2)
    means = np.array([[0, 0, 0, 0, 0, 100, 0, np.nan],
                      [0, 0, 0, 0, 0, 0, 0, 0],
                      [0.2, np.nextafter(np.float32(0.2), np.float32(1)), 1.0, 1.0, -1.0, 1.0, 2.0, 2.0]],
                     np.float32)
    N = means.shape[1]
    ls = np.full((3, N), -3.0, np.float32)
    q = np.tile(np.array([[1], [0], [0], [0]], np.float32), (1, N))
    q[:, 3] = 0.0  # degenerate quaternion
    lg = np.zeros(N, np.float32)
    lg[6] = np.inf  # non-finite logit
    sh = np.ones((3, N))
    sh[1, 1] = np.inf  # infinite colour
    sh[0, 2] = np.nan  # NaN colour clamps to 0 and stays visible
    sc = make_scene(means, ls, q, lg, sh, 0, [cam])
    rec = orc.preprocess(sc, cam)
    vis = rec["tiles"] > 0
    # 0: on the near plane; 1: just beyond but infinite colour; 2: fine (NaN colour -> 0);
    # 3: zero quaternion; 4: behind; 5: far off-screen; 6: infinite logit; 7: NaN mean
    assert list(vis) == [False, False, True, False, False, False, False, False]
    assert rec["rgb"][2, 0] == 0.0
    for g in np.nonzero(~vis)[0]:
        assert not rec["xyzo"][g].any() and not rec["conic"][g].any() and rec["radius"][g] == 0


def test_active_list_selects_records(orc):
    sc = S.make_config(0)
    cam = sc.cameras[0]
    full = orc.preprocess(sc, cam)
    act = np.arange(0, sc.N, 3, dtype=np.int32)
    sub = orc.preprocess(sc, cam, act, act.size)
    n = act.size
    for k in ("xyzo", "conic", "rgb", "radius", "rect", "tiles"):
        assert np.array_equal(sub[k][:n], full[k][act]), k
    assert not sub["tiles"][n:].any()


def test_fp32_spec_close_to_fp64(orc):
    sc = S.make_config(1)
    cam = sc.cameras[0]
    sub = np.arange(0, sc.N, 97)
    small = make_scene(sc.means[:, sub], sc.log_scales[:, sub], sc.quats[:, sub],
                       sc.opacity_logits[sub], sc.sh[:, sub], 3, [cam])
    rec = orc.preprocess(small, cam)
    out, vis, rad = orc.project_f64(params64(small), 3, small.N, cam)
    v = rec["tiles"] > 0
    assert np.array_equal(v, vis.astype(bool) & v)
    np.testing.assert_allclose(rec["xyzo"][v, :4], out[v, :4], rtol=1e-5, atol=1e-4)
    np.testing.assert_allclose(rec["rgb"][v, :3], out[v, 7:10], atol=1e-5)
    np.testing.assert_allclose(rec["conic"][v, :3], out[v, 4:7], rtol=1e-3,
                               atol=1e-4 * np.abs(out[v, 4:5]).max())
