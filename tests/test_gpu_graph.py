"""A whole multi-pose step captured as one CUDA graph (the bench's timed
loop): with the bin/sort in deferred mode no call reads the device from the
host, so the capture holds every launch; replaying it gives the images of
the direct calls bit for bit and the oracle's gradients within the suite's
tolerance, and the deferred result slots hold the last replay's counts."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, MultiViewRenderer, Rasterizer
from tests.gpu_helpers import assert_bits, grad_tol_check

pytestmark = pytest.mark.gpu

NAMES = ["means", "log_scales", "quats", "opacity_logits", "sh"]


def test_graph_replay_of_a_step_matches_direct_calls():
    sc = S.random_scene(3000, 160, 120, sh_degree=2, seed=160, n_poses=2, log_scale=(-2.2, 0.4))
    params = GaussianParams.from_scene(sc)
    cams = [gs.camera(c) for c in sc.cameras]
    gimg = [torch.from_numpy(sc.grad_image(p)).cuda() for p in range(2)]
    R = Rasterizer(sc.N, sc.sh_degree, sc.cameras[0].width, sc.cameras[0].height, capacity=64 * sc.N)

    def step(keep):
        for p, c in enumerate(cams):
            R.forward(params, c, sc.bg)
            g = R.backward(gimg[p])
            if keep is not None:
                keep.append((R.image.clone(), {k: v.clone() for k, v in g.items()}))

    direct = []
    step(direct)  # also loads every kernel before the capture
    torch.cuda.synchronize()
    R.deferred = True
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(None)
    slots = R._n_pending
    assert slots == 2
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    R._n_pending = slots
    counts = R.check()
    # the buffers hold the last pose of the last replay
    last = len(cams) - 1
    assert_bits(R.image.cpu().numpy(), direct[last][0].cpu().numpy(), "image after replay")
    ref = oracle.render(S.Scene(sc.name, sc.N, sc.sh_degree, sc.means, sc.log_scales, sc.quats,
                                sc.opacity_logits, sc.sh, [sc.cameras[last]], sc.bg, True))
    assert counts[last] == ref["bins"]["n_instances"]
    ob = oracle.backward(S.Scene(sc.name, sc.N, sc.sh_degree, sc.means, sc.log_scales, sc.quats,
                                 sc.opacity_logits, sc.sh, [sc.cameras[last]], sc.bg, True),
                         sc.cameras[last], ref["rec"], ref["bins"], sc.grad_image(last))
    for n in NAMES:
        grad_tol_check(R.grads[n].cpu().numpy(), ob["d_" + n], ob["m_" + n], what=f"{n} after replay")
    del graph


def test_graph_of_poses_on_their_own_streams():
    # one Rasterizer and stream per pose, forked from and joined to the
    # capture stream: each pose's replayed image equals its direct render
    sc = S.random_scene(2500, 144, 112, sh_degree=1, seed=161, n_poses=3, log_scale=(-2.2, 0.4))
    params = GaussianParams.from_scene(sc)
    cams = [gs.camera(c) for c in sc.cameras]
    gimg = [torch.from_numpy(sc.grad_image(p)).cuda() for p in range(3)]
    Rs = [Rasterizer(sc.N, sc.sh_degree, sc.cameras[0].width, sc.cameras[0].height, capacity=64 * sc.N)
          for _ in cams]
    streams = [torch.cuda.Stream() for _ in cams]

    def step():
        cur = torch.cuda.current_stream()
        for p, c in enumerate(cams):
            streams[p].wait_stream(cur)
            with torch.cuda.stream(streams[p]):
                Rs[p].forward(params, c, sc.bg)
                Rs[p].backward(gimg[p])
        for st in streams:
            cur.wait_stream(st)

    step()
    torch.cuda.synchronize()
    direct = [R.image.clone() for R in Rs]
    for R in Rs:
        R.deferred = True
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for R in Rs:
        R.image.zero_()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    for p, R in enumerate(Rs):
        R._n_pending = 1
        assert R.check()[0] > 0
        assert_bits(R.image.cpu().numpy(), direct[p].cpu().numpy(), f"image pose {p}")
    ref = oracle.render(S.Scene(sc.name, sc.N, sc.sh_degree, sc.means, sc.log_scales, sc.quats,
                                sc.opacity_logits, sc.sh, [sc.cameras[1]], sc.bg, True))
    assert_bits(Rs[1].image.cpu().numpy(), ref["fwd"]["image"], "pose 1 against the oracle")
    del graph


def test_graph_of_the_multiview_step():
    # the bench's step: one multi-view projection, the poses' sort and raster
    # work on their own streams, one multi-view backward; replayed images
    # equal the direct render bit for bit, and the replayed summed gradient
    # is within the suite's tolerance of the oracle's sum over the poses
    sc = S.random_scene(2500, 144, 112, sh_degree=3, seed=162, n_poses=3, log_scale=(-2.2, 0.4))
    params = GaussianParams.from_scene(sc)
    gimg = [torch.from_numpy(sc.grad_image(p)).cuda() for p in range(3)]
    mv = MultiViewRenderer(sc.N, sc.sh_degree, sc.cameras, capacity=64 * sc.N, n_streams=3)

    def step():
        mv.forward(params, sc.bg)
        mv.backward(gimg)

    step()
    torch.cuda.synchronize()
    direct = [R.image.clone() for R in mv.views]
    mv.set_deferred(True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for R in mv.views:
        R.image.zero_()
    for g in mv.grads.values():
        g.fill_(float("nan"))
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    for p, R in enumerate(mv.views):
        R._n_pending = 1
        assert R.check()[0] > 0
        assert_bits(R.image.cpu().numpy(), direct[p].cpu().numpy(), f"image pose {p}")
    ref_sum = {n: 0.0 for n in NAMES}
    mag_sum = {n: 0.0 for n in NAMES}
    for pose, cam in enumerate(sc.cameras):
        ref = oracle.render(sc, pose)
        ob = oracle.backward(sc, cam, ref["rec"], ref["bins"], sc.grad_image(pose))
        for n in NAMES:
            ref_sum[n] = ref_sum[n] + ob["d_" + n]
            mag_sum[n] = mag_sum[n] + ob["m_" + n]
    for n in NAMES:
        grad_tol_check(mv.grads[n].cpu().numpy(), ref_sum[n], mag_sum[n], what=f"{n} summed, after replay")
    del graph
