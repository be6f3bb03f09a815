"""Pins for the oracle's forward compositing.

References: the closed-form value of one isotropic Gaussian at the pixel
centres next to its mean; compositing invariants (1 - T equals the sum of
alpha * T; colour bounded by the colour range times 1 - T; no contributor means
background); per-pixel brute force over all Gaussians without tile lists; and
a float64 restatement of the per-pixel recursion on sampled pixels.
"""

import math

import numpy as np
import pytest

from differentiable_tile_rasterizer_b200 import synthetic as S
from tests._helpers import make_scene, simple_camera

C0 = 0.28209479177387814


def test_single_gaussian_closed_form(orc):
    W = H = 32
    f, z, s, logit, col = 40.0, 2.0, 0.02, 0.4, 0.7
    cam = simple_camera(W, H, f, cx=16.0, cy=16.0)
    k0 = (col - 0.5) / C0
    sc = make_scene([[0], [0], [z]], [[math.log(s)]] * 3, [[1], [0], [0], [0]], [logit],
                    [[k0], [k0], [k0]], 0, [cam])
    r = orc.render(sc)
    s_eff = math.exp(np.float64(np.float32(math.log(s))))
    sig2 = (f * s_eff / z) ** 2 + 0.3
    o = 1 / (1 + math.exp(-np.float64(np.float32(logit))))
    alpha = o * math.exp(-0.5 * (0.25 + 0.25) / sig2)
    img, T = r["fwd"]["image"], r["fwd"]["final_T"]
    for (v, u) in [(15, 15), (15, 16), (16, 15), (16, 16)]:
        assert img[0, v, u] == pytest.approx(alpha * col, rel=2e-6)
        assert T[v, u] == pytest.approx(1 - alpha, rel=2e-6)
        assert r["fwd"]["n_contrib"][v, u] == 1 and r["fwd"]["last"][v, u] == 1
    # one pixel further out along x: offset 1.5 instead of 0.5
    a2 = o * math.exp(-0.5 * (2.25 + 0.25) / sig2)
    assert img[1, 15, 17] == pytest.approx(a2 * col, rel=2e-6)


def _white_scene(seed, bg=(0, 0, 0)):
    sc = S.random_scene(400, 70, 50, sh_degree=0, seed=seed, bg=bg)
    sc.sh[:] = np.float32(math.sqrt(math.pi))  # colour C0*sqrt(pi) + 0.5 = 1
    return sc


def test_transmittance_telescopes(orc):
    sc = _white_scene(11)
    r = orc.render(sc)
    img, T = r["fwd"]["image"], r["fwd"]["final_T"]
    rgb = r["rec"]["rgb"][r["rec"]["tiles"] > 0, :3]
    assert np.abs(rgb - 1).max() < 1e-6
    # sum_k alpha_k T_k = 1 - T_final for unit colours
    assert np.abs(img - (1 - T)[None]).max() < 2e-5
    assert (r["fwd"]["n_contrib"] > 5).mean() > 0.3


def test_colour_bounds_and_background(orc):
    bg = np.array([0.2, 0.5, 0.9], np.float32)
    sc = S.random_scene(500, 61, 47, sh_degree=2, seed=12, bg=bg)
    r = orc.render(sc)
    f = r["fwd"]
    img, T, n = f["image"], f["final_T"], f["n_contrib"]
    rgb = r["rec"]["rgb"][r["rec"]["tiles"] > 0, :3]
    lo, hi = rgb.min(0), rgb.max(0)
    fg = img - T[None] * bg[:, None, None]
    for ch in range(3):
        assert np.all(fg[ch] <= hi[ch] * (1 - T) + 1e-5)
        assert np.all(fg[ch] >= lo[ch] * (1 - T) - 1e-5)
    empty = n == 0
    assert empty.any() and (~empty).any()
    assert np.all(T[empty] == 1) and np.all(img[:, empty] == bg[:, None])
    assert np.all(T >= 1e-4 * (1 - 0.99) * (1 - 1e-6))
    assert np.all(f["last"] >= n)


def test_stop_rule_is_inclusive(orc):
    sc = _white_scene(13)
    sc.opacity_logits[:] = 6.0  # opaque: pixels saturate quickly
    r = orc.render(sc)
    f = r["fwd"]
    stopped = f["final_T"] < 1e-4
    assert stopped.any()
    # a stopped pixel's last blend is the one that crossed: T before it >= 1e-4
    assert np.all(f["final_T"][stopped] >= 1e-4 * 0.01 * (1 - 1e-6))


def test_faint_gaussians_never_blend(orc):
    sc = S.random_scene(200, 48, 48, sh_degree=0, seed=14)
    sc.opacity_logits[:] = np.float32(-math.log(300.0 - 1.0))  # o = 1/300 < 1/255
    r = orc.render(sc)
    assert r["bins"]["n_instances"] > 0
    assert not r["fwd"]["n_contrib"].any()
    assert np.all(r["fwd"]["final_T"] == 1)


@pytest.mark.parametrize("which", ["tiny", "ragged", "deg3"])
def test_tiled_equals_bruteforce(orc, which):
    if which == "tiny":
        sc = S.make_config(0)
    elif which == "ragged":
        sc = S.random_scene(350, 83, 37, sh_degree=1, seed=15, bg=(0.1, 0.3, 0.2))
    else:
        sc = S.random_scene(250, 40, 40, sh_degree=3, seed=16)
    r = orc.render(sc)
    bf = orc.raster_fwd_bruteforce(r["rec"], r["cam"], sc.bg)
    for k in ("image", "final_T", "n_contrib", "last"):
        assert np.array_equal(bf[k], r["fwd"][k]), k


def test_float64_recursion_on_sampled_pixels(orc):
    sc = S.random_scene(300, 64, 64, sh_degree=1, seed=17, bg=(0.3, 0.1, 0.0))
    r = orc.render(sc)
    rec, b, f = r["rec"], r["bins"], r["fwd"]
    rng = np.random.default_rng(0)
    cam = r["cam"]
    checked = 0
    for _ in range(300):
        u, v = int(rng.integers(0, 64)), int(rng.integers(0, 64))
        t = (v // 16) * cam.tiles_x + u // 16
        s, e = b["ranges"][t]
        T, C, n, near = 1.0, np.zeros(3), 0, False
        for j in range(s, e):
            i = b["vals"][j]
            px, py, _, o = rec["xyzo"][i].astype(np.float64)
            A, B, Cc = rec["conic"][i, :3].astype(np.float64)
            dx, dy = px - (u + 0.5), py - (v + 0.5)
            a = min(0.99, o * math.exp(-0.5 * (A * dx * dx + Cc * dy * dy) - B * dx * dy))
            near |= abs(a - 1 / 255) < 1e-5 or abs(T * (1 - a) - 1e-4) < 1e-7
            if a < 1 / 255:
                continue
            C += a * T * rec["rgb"][i, :3]
            T *= 1 - a
            n += 1
            if T < 1e-4:
                break
        if near:
            continue
        checked += 1
        assert n == f["n_contrib"][v, u]
        assert T == pytest.approx(f["final_T"][v, u], rel=1e-4, abs=1e-9)
        np.testing.assert_allclose(C + T * sc.bg, f["image"][:, v, u], atol=2e-5)
    assert checked > 250


def test_tiled_equals_bruteforce_on_random_scenes(orc):
    # scene sizes, SH degrees, scale ranges and seeds drawn by hypothesis:
    # the tiled walk gives the brute-force composite bit for bit
    from hypothesis import given, settings
    from hypothesis import strategies as st

    @settings(max_examples=30, deadline=None)
    @given(st.integers(1, 160), st.integers(1, 70), st.integers(1, 50), st.integers(0, 3),
           st.sampled_from([(-3.5, 0.3), (-2.0, 0.5), (-1.0, 0.4)]), st.integers(0, 2 ** 16))
    def check(n, W, H, deg, log_scale, seed):
        sc = S.random_scene(n, W, H, sh_degree=deg, seed=seed, log_scale=log_scale)
        r = orc.render(sc)
        bf = orc.raster_fwd_bruteforce(r["rec"], r["cam"], sc.bg)
        for k in ("image", "final_T", "n_contrib", "last"):
            assert np.array_equal(bf[k], r["fwd"][k]), k

    check()
