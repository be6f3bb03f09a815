"""The bin/sort without a host round trip (gs_bin_sort_async, and the
Rasterizer's deferred mode built on it): the same keys, values and ranges as
the synchronous call and the oracle, and device-side reporting of the
capacity and look-back timeout failures with empty tile ranges."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, Rasterizer
from tests.gpu_helpers import assert_bits, gpu_forward, grad_tol_check

pytestmark = pytest.mark.gpu


def _prepared(sc, capacity=None, pose=0):
    cam = sc.cameras[pose]
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height, capacity=capacity)
    params = GaussianParams.from_scene(sc)
    c = gs.camera(cam)
    R.cull(params, c)
    R.preprocess(params, c)
    return R, c, params


def test_async_matches_oracle_bitexact():
    sc = S.random_scene(5000, 300, 200, sh_degree=1, seed=51, log_scale=(-1.5, 0.4))
    R, c, _ = _prepared(sc, capacity=600_000)  # ~544K instances
    res = torch.full((2,), -1, dtype=torch.int64, device="cuda")
    gs.gs_bin_sort_async(R._proj, R.N, c, R.offsets, R.keys, R.vals, R.capacity, R.ranges, res, R.sort_ws)
    torch.cuda.synchronize()
    ni, st = res.tolist()
    ref = oracle.render(sc)
    assert st == gs.GS_OK and ni == ref["bins"]["n_instances"] > 4096
    R.n_instances = ni
    b = R.bins_numpy()
    for k in ("offsets", "keys", "vals", "ranges"):
        assert_bits(b[k], ref["bins"][k], k)


def test_deferred_views_match_checked_views():
    sc = S.random_scene(4000, 256, 192, sh_degree=2, seed=52, n_poses=3, log_scale=(-1.5, 0.4))
    params = GaussianParams.from_scene(sc)
    cam = sc.cameras[0]
    Rd = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height, capacity=400_000)  # <= ~350K per view
    Rd.deferred = True
    Rs = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height, capacity=400_000)
    out = []
    for p in range(3):
        Rd.forward(params, sc.cameras[p], sc.bg)
        g = torch.from_numpy(sc.grad_image(p)).cuda()
        Rd.backward(g)
        out.append((Rd.image.clone(), Rd.final_T.clone(), {k: v.clone() for k, v in Rd.grads.items()}))
    counts = Rd.check()
    assert Rd.check() == []  # nothing pending any more
    for p in range(3):
        Rs.forward(params, sc.cameras[p], sc.bg)
        Rs.backward(torch.from_numpy(sc.grad_image(p)).cuda())
        torch.cuda.synchronize()
        assert counts[p] == Rs.n_instances
        assert_bits(out[p][0].cpu().numpy(), Rs.image.cpu().numpy(), f"image {p}")
        assert_bits(out[p][1].cpu().numpy(), Rs.final_T.cpu().numpy(), f"T {p}")
        # same kernels on the same inputs; only the order of the fp32 atomic
        # sums differs, so both runs are held to the oracle's gradients with
        # the suite's tolerance (relative plus a floor from the summed magnitudes)
        sub = S.Scene(sc.name, sc.N, sc.sh_degree, sc.means, sc.log_scales, sc.quats, sc.opacity_logits, sc.sh,
                      [sc.cameras[p]], sc.bg, True)
        ref = oracle.render(sub)
        ob = oracle.backward(sub, sub.cameras[0], ref["rec"], ref["bins"], sc.grad_image(p))
        for k, v in Rs.grads.items():
            grad_tol_check(out[p][2][k].cpu().numpy(), ob["d_" + k], ob["m_" + k], what=f"deferred {k} {p}")
            grad_tol_check(v.cpu().numpy(), ob["d_" + k], ob["m_" + k], what=f"checked {k} {p}")


def test_deferred_capacity_failure_leaves_tiles_empty_then_recovers():
    sc = S.random_scene(3000, 128, 128, sh_degree=0, seed=37, log_scale=(-1.5, 0.3))
    R, c, _ = _prepared(sc, capacity=16)
    R.deferred = True
    R.bin_sort(c)
    R.raster_fwd(c, sc.bg)  # reads no list entries
    torch.cuda.synchronize()
    assert not R.ranges.any()
    assert not R.n_contrib.any()
    with pytest.raises(gs.GsError) as ei:
        R.check()
    assert ei.value.status == gs.GS_ERR_CAPACITY
    ref = oracle.render(sc)
    assert R.capacity > ref["bins"]["n_instances"] > 16  # grown for the count seen
    R.bin_sort(c)
    assert R.check() == [ref["bins"]["n_instances"]]
    assert_bits(R.bins_numpy()["keys"], ref["bins"]["keys"], "keys after growth")


def test_async_lookback_timeout_reported_in_result():
    sc = S.random_scene(12000, 256, 256, sh_degree=0, seed=42, log_scale=(-1.5, 0.3))
    R = gpu_forward(sc)
    assert int((R.rec["tiles"] > 0).sum()) > 4096 and R.n_instances > 3 * 4096  # several sort tiles per pass
    c = gs.camera(sc.cameras[0])
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    gs.gs_debug_set_stalled_sort_tile(1)
    try:
        gs.gs_bin_sort_async(R._proj, R.N, c, None, R.keys, R.vals, R.capacity, R.ranges, res, R.sort_ws)
        torch.cuda.synchronize()
    finally:
        gs.gs_debug_set_stalled_sort_tile(-1)
    assert res[1].item() == gs.GS_ERR_DEVICE_TIMEOUT
    assert not R.ranges.any()
    gs.gs_bin_sort_async(R._proj, R.N, c, None, R.keys, R.vals, R.capacity, R.ranges, res, R.sort_ws)
    torch.cuda.synchronize()
    assert res.tolist() == [R.n_instances, gs.GS_OK]
    ref = oracle.render(sc)
    R.n_instances = int(res[0].item())
    assert_bits(R.bins_numpy()["keys"], ref["bins"]["keys"], "keys after recovery")
