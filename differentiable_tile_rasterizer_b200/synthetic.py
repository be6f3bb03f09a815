"""Seeded synthetic workloads for the Gaussian-splat rasterizer.

This module only draws inputs: Gaussian parameters, camera poses, upstream
image gradients. It holds none of the rasterizer's arithmetic, so both the CUDA
path and the CPU oracle may consume what it produces.

Five workloads are defined, following the problem statement of the
differentiable tile rasterizer (3D Gaussian splatting) and its stated sizes:

  0  tiny:  256 Gaussians, 64x64, SH degree 0, forward only
  1  small: 100K Gaussians, 800x800, SH degree 3, forward + backward
  2  1080p: 1M Gaussians, 1920x1080, SH degree 3, 4 poses, forward + backward
  3  city:  6M Gaussians in 500 clusters, importance weights, LOD 800,
            importance quantile 0.3, 1920x1080, forward + backward
  4  4K:    10M Gaussians, 3840x2160, SH degree 3, 8 poses, forward only

Layouts (structure of arrays, float32, C-contiguous):
  means [3][N], log_scales [3][N], quats [4][N] as (w, x, y, z),
  opacity_logits [N], sh [K*3][N] with plane index k*3 + channel,
  importance [N] (only workload 3).

Cameras follow the pinhole model with OpenCV axes (x right, y down, z
forward); R, t map world to camera, campos is the camera centre in world
coordinates. Pixel (u, v) is sampled at (u + 0.5, v + 0.5).
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

SQRT_PI = math.sqrt(math.pi)


@dataclasses.dataclass
class Camera:
    R: np.ndarray          # (3, 3) float32, world -> camera rotation, row-major
    t: np.ndarray          # (3,) float32, world -> camera translation
    campos: np.ndarray     # (3,) float32, camera centre in world coordinates
    fx: float
    fy: float
    cx: float
    cy: float
    width: int
    height: int
    near_z: float = 0.2

    @property
    def tiles_x(self) -> int:
        return (self.width + 15) // 16

    @property
    def tiles_y(self) -> int:
        return (self.height + 15) // 16


@dataclasses.dataclass
class Scene:
    name: str
    N: int
    sh_degree: int
    means: np.ndarray
    log_scales: np.ndarray
    quats: np.ndarray
    opacity_logits: np.ndarray
    sh: np.ndarray
    cameras: List[Camera]
    bg: np.ndarray
    backward: bool
    importance: Optional[np.ndarray] = None
    lod_dist: float = 0.0          # <= 0 disables the distance gate
    importance_q: float = 0.0      # 0 disables the importance mask
    seed: int = 0

    @property
    def K(self) -> int:
        return (self.sh_degree + 1) ** 2

    def grad_image(self, pose: int) -> np.ndarray:
        """Upstream dL/dimage for one pose: N(0, 1), shape [3][H][W], float32."""
        cam = self.cameras[pose]
        rng = np.random.default_rng([self.seed, 1000 + pose])
        return rng.standard_normal((3, cam.height, cam.width), dtype=np.float32)


def look_at(eye, target, up, fx, fy, cx, cy, width, height, near_z=0.2) -> Camera:
    """Camera at `eye` looking at `target`; image 'down' is -up."""
    eye = np.asarray(eye, dtype=np.float64)
    f = np.asarray(target, dtype=np.float64) - eye
    f /= np.linalg.norm(f)
    r = np.cross(f, np.asarray(up, dtype=np.float64))
    r /= np.linalg.norm(r)
    d = np.cross(f, r)
    R = np.stack([r, d, f]).astype(np.float64)
    t = -R @ eye
    return Camera(R=R.astype(np.float32), t=t.astype(np.float32),
                  campos=eye.astype(np.float32), fx=float(fx), fy=float(fy),
                  cx=float(cx), cy=float(cy), width=int(width),
                  height=int(height), near_z=float(near_z))


def _unit_quats(rng, n):
    q = rng.standard_normal((4, n), dtype=np.float32)
    q /= np.sqrt((q.astype(np.float64) ** 2).sum(0)).astype(np.float32)
    return np.ascontiguousarray(q)


def _sh_planes(rng, n, K, dc_kind):
    sh = np.empty((K * 3, n), dtype=np.float32)
    if dc_kind == "rgb01":
        # Colour = C0*k + 0.5 is U(0,1) when k is U(-sqrt(pi), sqrt(pi)).
        sh[0:3] = rng.uniform(-SQRT_PI, SQRT_PI, (3, n)).astype(np.float32)
    else:
        sh[0:3] = rng.random((3, n), dtype=np.float32)
    if K > 1:
        sh[3:] = rng.normal(0.0, 0.1, (3 * (K - 1), n)).astype(np.float32)
    return sh


def random_scene(N, width, height, sh_degree=0, seed=0, n_poses=1, backward=True,
                 mean_box=1.0, cam_dist=3.0, focal=None, log_scale=(-3.0, 0.5),
                 opacity=(0.0, 1.0), with_importance=False, lod_dist=0.0,
                 importance_q=0.0, bg=(0.0, 0.0, 0.0), name=None) -> Scene:
    """A small random scene for parity tests (ragged sizes allowed)."""
    rng = np.random.default_rng(seed)
    K = (sh_degree + 1) ** 2
    means = rng.uniform(-mean_box, mean_box, (3, N)).astype(np.float32)
    log_scales = rng.normal(log_scale[0], log_scale[1], (3, N)).astype(np.float32)
    quats = _unit_quats(rng, N)
    logits = rng.normal(opacity[0], opacity[1], N).astype(np.float32)
    sh = _sh_planes(rng, N, K, "rgb01" if sh_degree == 0 else "dc01")
    focal = focal if focal is not None else float(max(width, height))
    cams = []
    for p in range(n_poses):
        ang = 2.0 * math.pi * p / max(n_poses, 1)
        eye = (cam_dist * math.sin(ang), 0.3 * p, -cam_dist * math.cos(ang))
        cams.append(look_at(eye, (0, 0, 0), (0, -1, 0), focal, focal,
                            width / 2.0, height / 2.0, width, height))
    imp = rng.exponential(1.0, N).astype(np.float32) if with_importance else None
    return Scene(name or f"random{N}_{width}x{height}_sh{sh_degree}", N, sh_degree,
                 means, log_scales, quats, logits, sh, cams,
                 np.asarray(bg, np.float32), backward, imp, lod_dist, importance_q, seed)


def make_config(idx: int) -> Scene:
    """The five stated workloads; seed = workload index."""
    rng = np.random.default_rng(idx)
    if idx == 0:
        N, K = 256, 1
        means = rng.uniform(-1, 1, (3, N)).astype(np.float32)
        log_scales = rng.normal(-3.0, 0.5, (3, N)).astype(np.float32)
        quats = _unit_quats(rng, N)
        logits = rng.normal(0.0, 1.0, N).astype(np.float32)
        sh = _sh_planes(rng, N, K, "rgb01")
        cam = Camera(R=np.eye(3, dtype=np.float32), t=np.array([0, 0, 3], np.float32),
                     campos=np.array([0, 0, -3], np.float32), fx=64.0, fy=64.0,
                     cx=32.0, cy=32.0, width=64, height=64)
        return Scene("tiny_256_64x64_sh0", N, 0, means, log_scales, quats, logits,
                     sh, [cam], np.zeros(3, np.float32), False, seed=idx)
    if idx == 1:
        N, K = 100_000, 16
        means = rng.standard_normal((3, N), dtype=np.float32)
        log_scales = rng.normal(-3.0, 0.5, (3, N)).astype(np.float32)
        quats = _unit_quats(rng, N)
        logits = rng.normal(0.0, 1.0, N).astype(np.float32)
        sh = _sh_planes(rng, N, K, "dc01")
        cam = look_at((4, 0, 0), (0, 0, 0), (0, 0, 1), 1000, 1000, 400, 400, 800, 800)
        return Scene("100k_800x800_sh3", N, 3, means, log_scales, quats, logits, sh,
                     [cam], np.zeros(3, np.float32), True, seed=idx)
    if idx == 2:
        N, K = 1_000_000, 16
        n_surf = int(0.7 * N)
        means = np.empty((3, N), np.float32)
        xy = rng.uniform(-5, 5, (2, n_surf)).astype(np.float32)
        z = (np.sin(xy[0].astype(np.float64)) * np.cos(xy[1].astype(np.float64))
             + rng.normal(0, 0.1, n_surf))
        means[0:2, :n_surf] = xy
        means[2, :n_surf] = z.astype(np.float32)
        means[:, n_surf:] = rng.uniform(-5, 5, (3, N - n_surf)).astype(np.float32)
        log_scales = rng.normal(-4.0, 0.7, (3, N)).astype(np.float32)
        quats = _unit_quats(rng, N)
        logits = rng.normal(0.0, 1.0, N).astype(np.float32)
        sh = _sh_planes(rng, N, K, "dc01")
        cams = []
        while len(cams) < 4:
            u = rng.standard_normal(3)
            u /= np.linalg.norm(u)
            if abs(u[2]) > 0.9:
                continue
            cams.append(look_at(15.0 * u, (0, 0, 0), (0, 0, 1), 1400, 1400, 960, 540,
                                1920, 1080))
        return Scene("1m_1920x1080_sh3_4poses", N, 3, means, log_scales, quats, logits,
                     sh, cams, np.zeros(3, np.float32), True, seed=idx)
    if idx == 3:
        n_clusters, per = 500, 12_000
        N, K = n_clusters * per, 16
        centres = rng.uniform([0, 0, 0], [2000, 2000, 100], (n_clusters, 3))
        means = np.empty((3, N), np.float32)
        for c in range(n_clusters):
            pts = centres[c][:, None] + 20.0 * rng.standard_normal((3, per))
            means[:, c * per:(c + 1) * per] = pts.astype(np.float32)
        log_scales = rng.normal(-3.0, 0.5, (3, N)).astype(np.float32)
        quats = _unit_quats(rng, N)
        logits = rng.normal(0.0, 1.0, N).astype(np.float32)
        sh = _sh_planes(rng, N, K, "dc01")
        importance = rng.exponential(1.0, N).astype(np.float32)
        eye = np.array([1000.0, 1000.0, 300.0])
        cam = look_at(eye, eye + np.array([0.0, 1.0, -1.0]), (0, 0, 1), 1400, 1400,
                      960, 540, 1920, 1080)
        return Scene("city_6m_1920x1080_sh3", N, 3, means, log_scales, quats, logits, sh,
                     [cam], np.zeros(3, np.float32), True, importance,
                     lod_dist=800.0, importance_q=0.3, seed=idx)
    if idx == 4:
        N, K = 10_000_000, 16
        means = (2.0 * rng.standard_normal((3, N), dtype=np.float32)).astype(np.float32)
        log_scales = rng.normal(-5.0, 0.8, (3, N)).astype(np.float32)
        quats = _unit_quats(rng, N)
        logits = rng.normal(-1.0, 1.0, N).astype(np.float32)
        sh = _sh_planes(rng, N, K, "dc01")
        cams = []
        for k in range(8):
            a = 2.0 * math.pi * k / 8
            cams.append(look_at((6 * math.cos(a), 6 * math.sin(a), 0.0), (0, 0, 0),
                                (0, 0, 1), 2800, 2800, 1920, 1080, 3840, 2160))
        return Scene("10m_3840x2160_sh3_8poses", N, 3, means, log_scales, quats, logits,
                     sh, cams, np.zeros(3, np.float32), False, seed=idx)
    raise ValueError(f"unknown workload {idx}")


CONFIG_NAMES = {
    0: "tiny_256_64x64_sh0",
    1: "100k_800x800_sh3",
    2: "1m_1920x1080_sh3_4poses",
    3: "city_6m_1920x1080_sh3",
    4: "10m_3840x2160_sh3_8poses",
}
