"""Small hand-built scenes and comparison helpers shared by the tests."""

import numpy as np

from differentiable_tile_rasterizer_b200 import synthetic as S


def simple_camera(W=64, H=48, f=50.0, cx=None, cy=None, near=0.2):
    """Camera at the origin looking down +z with R = I."""
    return S.Camera(R=np.eye(3, dtype=np.float32), t=np.zeros(3, np.float32),
                    campos=np.zeros(3, np.float32), fx=f, fy=f,
                    cx=W / 2.0 if cx is None else cx, cy=H / 2.0 if cy is None else cy,
                    width=W, height=H, near_z=near)


def make_scene(means, log_scales, quats, logits, sh, sh_degree, cams, bg=(0, 0, 0),
               backward=True, importance=None, lod_dist=0.0, importance_q=0.0, name="custom"):
    means = np.ascontiguousarray(np.asarray(means, np.float32).reshape(3, -1))
    N = means.shape[1]
    K = (sh_degree + 1) ** 2
    return S.Scene(name, N, sh_degree, means,
                   np.ascontiguousarray(np.asarray(log_scales, np.float32).reshape(3, N)),
                   np.ascontiguousarray(np.asarray(quats, np.float32).reshape(4, N)),
                   np.ascontiguousarray(np.asarray(logits, np.float32).reshape(N)),
                   np.ascontiguousarray(np.asarray(sh, np.float32).reshape(3 * K, N)),
                   list(cams), np.asarray(bg, np.float32), backward,
                   None if importance is None else np.asarray(importance, np.float32),
                   lod_dist, importance_q)


def params64(scene):
    return tuple(np.asarray(a, np.float64).copy() for a in
                 (scene.means, scene.log_scales, scene.quats, scene.opacity_logits, scene.sh))


def grad_close(got, ref, mag, rtol=1e-3, mtol=1e-4):
    """Elementwise |got - ref| <= rtol |ref| + mtol * mag; returns (ok, worst ratio)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    mag = np.asarray(mag, np.float64)
    bound = rtol * np.abs(ref) + mtol * mag + 1e-30
    ratio = np.abs(got - ref) / bound
    return bool(np.all(ratio <= 1.0)), float(ratio.max(initial=0.0))
