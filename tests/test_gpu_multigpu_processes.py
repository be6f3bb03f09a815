"""The index-interleaved render through render_distributed in real
processes: two ranks, each its own process on the same GPU, joined by a gloo
group whose all-to-alls run on host copies of the exchanged tensors. No
kernel of one rank waits on the other's; the ranks meet only in the host
collectives. The image composed from the ranks' bands is the oracle's bit for
bit, and the parameter gradients gathered from the ranks are within the
suite's gradient tolerance of the oracle's. After each pose the ranks
rebalance their tile-row bands by the work measured per row; the bands change
no output bit."""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
from differentiable_tile_rasterizer_b200 import synthetic as S
from tests.gpu_helpers import assert_bits, grad_tol_check

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NAMES = ["means", "log_scales", "quats", "opacity_logits", "sh"]


def _scene():
    return S.random_scene(3000, 160, 128, sh_degree=2, seed=140, log_scale=(-2.2, 0.5), n_poses=2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from differentiable_tile_rasterizer_b200.multigpu import (DistExchange, InterleavedRank, balance_bands,
                                                             local_params, render_distributed)
    from differentiable_tile_rasterizer_b200.pipeline import GaussianParams
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        sc = _scene()
        lp = local_params(GaussianParams.from_scene(sc), rank, world)
        ex = DistExchange(host_staging=True)
        cam0 = sc.cameras[0]
        rk = InterleavedRank(lp.N, sc.sh_degree, cam0.width, cam0.height, rank, world)
        for pose in range(len(sc.cameras)):
            cam = sc.cameras[pose]
            g = torch.from_numpy(sc.grad_image(pose)).cuda()
            img, grads = render_distributed(rk, ex, lp, cam, sc.bg, g)
            torch.cuda.synchronize()
            lo, hi = rk.row_lo * 16, min(rk.row_hi * 16, cam.height)
            np.savez(os.path.join(out_dir, f"r{rank}_p{pose}.npz"), lo=lo, hi=hi, img=img[:, lo:hi].cpu().numpy(),
                     **{n: grads[n].cpu().numpy() for n in NAMES})
            # the next pose's bands balance this pose's measured work per row
            rk.set_bands(balance_bands(ex.row_costs(rk.band_row_costs()), world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_render_distributed_two_processes_gloo(tmp_path):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(600)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    sc = _scene()
    for pose in range(len(sc.cameras)):
        cam = sc.cameras[pose]
        sub = S.Scene(sc.name, sc.N, sc.sh_degree, sc.means, sc.log_scales, sc.quats, sc.opacity_logits, sc.sh,
                      [cam], sc.bg, True)
        ref = oracle.render(sub)
        parts = [np.load(os.path.join(tmp_path, f"r{r}_p{pose}.npz")) for r in range(world)]
        img = np.zeros_like(ref["fwd"]["image"])
        covered = np.zeros(cam.height, bool)
        for d in parts:
            lo, hi = int(d["lo"]), int(d["hi"])
            img[:, lo:hi] = d["img"]
            covered[lo:hi] = True
        assert covered.all()
        assert_bits(img, ref["fwd"]["image"], f"composed image pose {pose}")
        ob = oracle.backward(sub, cam, ref["rec"], ref["bins"], sc.grad_image(pose))
        for n in NAMES:
            full = np.zeros(ob["d_" + n].shape, np.float32)
            for r, d in enumerate(parts):
                full[..., r::world] = d[n]
            grad_tol_check(full, ob["d_" + n], ob["m_" + n], what=f"{n} pose {pose}")
