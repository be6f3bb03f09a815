"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the oracle."""

import os

import numpy as np
import torch

from differentiable_tile_rasterizer_b200 import gs
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, Rasterizer


def gpu_forward(scene, pose=0, capacity=None):
    cam = scene.cameras[pose]
    params = GaussianParams.from_scene(scene)
    R = Rasterizer(scene.N, scene.sh_degree, cam.width, cam.height, capacity=capacity)
    R.want_offsets = True
    R.forward(params, cam, scene.bg, scene.lod_dist, scene.importance_q)
    torch.cuda.synchronize()
    return R


def fwd_numpy(R):
    return {"image": R.image.cpu().numpy(), "final_T": R.final_T.cpu().numpy(),
            "n_contrib": R.n_contrib.cpu().numpy(), "last": R.last.cpu().numpy()}


def load_records(R, rec):
    """Overwrite the rasterizer's record buffers with (oracle) numpy records."""
    n = rec["tiles"].shape[0]
    for k in ("xyzo", "conic", "rgb"):
        R.rec[k][:n].copy_(torch.from_numpy(np.ascontiguousarray(rec[k])))
    R.rec["radius"][:n].copy_(torch.from_numpy(rec["radius"]))
    R.rec["rect"][:n].copy_(torch.from_numpy(np.ascontiguousarray(rec["rect"]).view(np.int16)))
    R.rec["tiles"][:n].copy_(torch.from_numpy(rec["tiles"]))


def load_bins(R, bins):
    I = bins["n_instances"]
    R._ensure_capacity(max(I, 1))
    if I:
        R.keys[:I].copy_(torch.from_numpy(bins["keys"].view(np.int64)))
        R.vals[:I].copy_(torch.from_numpy(bins["vals"].view(np.int32)))
    R.ranges.copy_(torch.from_numpy(np.ascontiguousarray(bins["ranges"]).view(np.int32).reshape(-1, 2)))
    R.n_instances = I


def bits_equal(a, b):
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    if a.dtype == np.float32:
        a, b = a.view(np.uint32), b.view(np.uint32)
    return np.array_equal(a, b), int(np.count_nonzero(a != b)) if a.shape == b.shape else -1


def assert_bits(a, b, what):
    ok, n = bits_equal(a, b)
    assert ok, f"{what}: {n} elements differ"


# Floors m of the gradient tolerance |g - g_ref| <= rtol |g_ref| + m S whose
# worst ratios every check records: 1e-5 is the floor of the stated contract
# (1e-3 relative plus 1e-5 of the magnitude sum S), 1e-4 a looser one kept
# for comparison.
FLOORS = (1e-5, 1e-4)
# What the checks enforce unless a test passes its own mtol.
GRAD_FLOOR = 1e-5
# (what, elements, worst ratio at each floor of FLOORS), one row per check,
# printed by the terminal summary of tests/conftest.py.
GRAD_RATIOS = []


def grad_ratio(got, ref, mag, rtol, mtol):
    """Elementwise |got - ref| / (rtol |ref| + mtol mag) as float64."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(got - ref) / (rtol * np.abs(ref) + mtol * np.asarray(mag, np.float64) + 1e-30)


def grad_tol_check(got, ref, mag, rtol=1e-3, mtol=None, what=""):
    """Asserts |got - ref| <= rtol |ref| + mtol S elementwise (mtol defaults
    to GRAD_FLOOR) and records the worst ratio at every floor of FLOORS."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    mag = np.asarray(mag, np.float64)
    if mtol is None:
        mtol = GRAD_FLOOR
    worst = tuple(float(grad_ratio(got, ref, mag, rtol, m).max(initial=0.0)) for m in FLOORS)
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0].split("::")[-1]
    GRAD_RATIOS.append((f"{test} {what}".strip(), int(ref.size), rtol, worst))
    ratio = grad_ratio(got, ref, mag, rtol, mtol)
    bad = ratio > 1.0
    if bad.any():
        i = int(np.argmax(ratio))
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst at {np.unravel_index(i, ref.shape)}:"
                             f" got {got.flat[i]} ref {ref.flat[i]} mag {mag.flat[i]}")
