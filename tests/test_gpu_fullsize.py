"""Parity at the stated full sizes, in the configuration bench.py times.

The oracle computes the records, keys and ranges of a whole view, the image,
final T, contributor counts and last indices of every pixel of the frame, and
the gradients. Integer results must be bit-exact, floats of the specification
bit-equal (within 1e-4), gradients within the suite's tolerance (see
test_gpu_parity).
"""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, MultiViewRenderer, Rasterizer
from tests.gpu_helpers import assert_bits, grad_tol_check

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

NAMES = ["means", "log_scales", "quats", "opacity_logits", "sh"]
COLS = [0, 1, 4, 5, 6, 2, 8, 9, 10]  # grad2d layout -> (px, py, A, B, C, o, r, g, b)


def _render(sc, pose, backward):
    cam = sc.cameras[pose]
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height, capacity=6 * sc.N)  # as bench.py
    R.want_offsets = True
    params = GaussianParams.from_scene(sc)
    R.forward(params, cam, sc.bg, sc.lod_dist, sc.importance_q)
    g = None
    if backward:
        g = sc.grad_image(pose)
        R.backward(torch.from_numpy(g).cuda())
    torch.cuda.synchronize()
    return R, g


def _check_forward(sc, pose, R):
    """Cull, records, keys, order and ranges, then every pixel of the frame."""
    cam = sc.cameras[pose]
    use_cull = sc.lod_dist > 0 or sc.importance_q > 0
    cl = oracle.cull(sc, cam)
    if use_cull:
        assert_bits(R.mask.cpu().numpy(), cl["mask"], "mask")
        na = cl["n_active"]
        assert int(R.n_active.item()) == na
        assert_bits(R.active_idx[:na].cpu().numpy(), cl["active_idx"], "active_idx")
    rec = oracle.preprocess(sc, cam, cl["active_idx"] if use_cull else None, cl["n_active"] if use_cull else None)
    got = R.records_numpy()
    for k in ("xyzo", "conic", "rgb", "radius", "rect", "tiles"):
        assert_bits(got[k], rec[k], k)
    bins = oracle.bin_sort(rec, cam)
    b = R.bins_numpy()
    assert b["n_instances"] == bins["n_instances"]
    for k in ("offsets", "keys", "vals", "ranges"):
        assert_bits(b[k], bins[k], k)
    f = oracle.raster_fwd(rec, bins, cam, sc.bg)
    assert_bits(R.n_contrib.cpu().numpy(), f["n_contrib"], f"n_contrib pose {pose}")
    assert_bits(R.last.cpu().numpy(), f["last"], f"last pose {pose}")
    assert_bits(R.final_T.cpu().numpy(), f["final_T"], f"final_T pose {pose}")
    assert_bits(R.image.cpu().numpy(), f["image"], f"image pose {pose}")
    assert int(f["n_contrib"].astype(np.int64).sum()) > 0
    return rec, bins


def test_1m_1080p_sh3_bench_workload_pose0():
    sc = S.make_config(2)
    R, g = _render(sc, 0, backward=True)
    rec, bins = _check_forward(sc, 0, R)
    ob = oracle.backward(sc, sc.cameras[0], rec, bins, g)
    na = rec["n_active"]
    grad_tol_check(R.grad2d.cpu().numpy()[:na][:, COLS], ob["g2d"], ob["s2d"], what="grad2d")
    for n in NAMES:
        grad_tol_check(R.grads[n].cpu().numpy(), ob["d_" + n], ob["m_" + n], what=n)


def test_1m_1080p_sh3_importance_pass_pose0():
    # importance weights of the whole view, every Gaussian (tolerance as in
    # test_gpu_importance: the fp32 summation tree of positive terms)
    sc = S.make_config(2)
    cam = sc.cameras[0]
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height, capacity=6 * sc.N)
    imp = torch.zeros(sc.N, dtype=torch.float32, device="cuda")
    R.forward_importance(GaussianParams.from_scene(sc), cam, imp, sc.bg)
    torch.cuda.synchronize()
    got = imp.cpu().numpy().astype(np.float64)
    rec = oracle.preprocess(sc, cam)
    bins = oracle.bin_sort(rec, cam)
    ref = oracle.importance(rec, bins, cam, sc.N)
    bound = (6.0 + 4.0 * rec["tiles"]) * 2.0 ** -23 * ref + 1e-30
    bad = np.abs(got - ref) > bound
    assert not bad.any(), (bad.sum(), got[bad][:3], ref[bad][:3])
    assert ref.sum() > 1e5


def test_1m_1080p_sh3_bench_workload_other_poses_forward():
    # the other three poses of the bench step, every pixel
    sc = S.make_config(2)
    for pose in (1, 2, 3):
        R, _ = _render(sc, pose, backward=False)
        _check_forward(sc, pose, R)


def test_city_6m_cull_and_backward():
    sc = S.make_config(3)
    R, g = _render(sc, 0, backward=True)
    rec, bins = _check_forward(sc, 0, R)
    cam = sc.cameras[0]
    na = rec["n_active"]
    assert 0 < na < sc.N
    ob = oracle.backward(sc, cam, rec, bins, g, params3d=False)
    grad_tol_check(R.grad2d.cpu().numpy()[:na][:, COLS], ob["g2d"], ob["s2d"], what="grad2d")
    # parameter gradients on a sample of the active Gaussians (the oracle's full
    # N-sized fp64 outputs would need ~6 GB of host memory)
    rng = np.random.default_rng(1)
    pos = np.sort(rng.choice(na, 20_000, replace=False))
    gid = rec["active_idx"][pos]
    sub = S.Scene("city_sample", pos.size, 3, sc.means[:, gid], sc.log_scales[:, gid], sc.quats[:, gid],
                  sc.opacity_logits[gid], sc.sh[:, gid], [cam], sc.bg, True)
    sub_rec = {k: (v[pos] if isinstance(v, np.ndarray) and v.shape[:1] == (sc.N,) else v) for k, v in rec.items()}
    sub_rec["active_idx"] = None
    sub_rec["n_active"] = pos.size
    ref = oracle.preprocess_bwd(sub, cam, sub_rec, ob["g2d"][pos])
    # magnitude bound: the sums of absolute per-pixel contributions propagated
    # through the chain, as oracle.backward forms it for whole views
    mag = oracle.preprocess_bwd(sub, cam, sub_rec, ob["s2d"][pos])
    for n in NAMES:
        got = R.grads[n].cpu().numpy()[..., gid]
        grad_tol_check(got, ref["d_" + n], mag["m_" + n], what=n)
    # culled Gaussians have zero gradients
    culled = ~R.mask.cpu().numpy().astype(bool)
    for n in NAMES:
        assert not R.grads[n].cpu().numpy()[..., culled].any()


def test_10m_4k_sh3_forward_two_poses():
    sc = S.make_config(4)
    for pose in (0, 5):
        R, _ = _render(sc, pose, backward=False)
        _check_forward(sc, pose, R)
        del R
        torch.cuda.empty_cache()


def test_10m_4k_sh3_multiview_all_eight_poses():
    # one parameter pass for the 8 views; views 2 and 7 checked in full
    # (records, sort and every pixel)
    sc = S.make_config(4)
    mv = MultiViewRenderer(sc.N, sc.sh_degree, sc.cameras, capacity=6 * sc.N)
    for R in mv.views:
        R.want_offsets = True
    mv.forward(GaussianParams.from_scene(sc), sc.bg)
    torch.cuda.synchronize()
    for pose in (2, 7):
        _check_forward(sc, pose, mv.views[pose])
    del mv
    torch.cuda.empty_cache()
