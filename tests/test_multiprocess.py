"""The multi-process host logic of bench.py on CPU (gloo, world size 2): the
path runs as independent replicas, so the only cross-rank steps are the
barrier and the max over ranks of the device times; under torchrun the
reference arm prints one JSON line from rank 0 only."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(world)
        got = bench._max_over_ranks(10.0 + 5.0 * rank, world)
        out.put((rank, got))
        bench._barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    assert res == {0: 15.0, 1: 15.0}


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--ref-tile-stride", "512"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def _exchange_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from differentiable_tile_rasterizer_b200.multigpu import DistExchange
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ex = DistExchange()
        # rank r sends (r + 1) * (q + 1) rows of 3 values to rank q, each row
        # tagged (source, destination, row)
        counts = [(rank + 1) * (q + 1) for q in range(world)]
        rows = [torch.tensor([rank, q, k], dtype=torch.int64) for q in range(world) for k in range(counts[q])]
        send = torch.stack(rows).reshape(-1)
        recv_counts = ex.counts(counts, "cpu")
        recv = ex.payload(send, counts, recv_counts, 3).reshape(-1, 3)
        # the single-read form: the counts exchanged before they are read
        s2, r2 = DistExchange(host_staging=True).counts_from_device(torch.tensor(counts, dtype=torch.int64))
        assert s2 == counts and r2 == recv_counts
        # band row costs: every rank fills its own rows, all get the sum
        import numpy as np
        local = np.zeros(5)
        local[rank] = rank + 1.0
        assert DistExchange(host_staging=True).row_costs(local).tolist() == [1.0, 2.0, 3.0, 0.0, 0.0]
        out.put((rank, recv_counts, recv.tolist()))
    finally:
        dist.destroy_process_group()


def test_exchange_counts_and_payload_with_gloo():
    world, port = 3, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_exchange_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = {r: (c, rows) for r, c, rows in (q.get(timeout=10) for _ in range(world))}
    for dst in range(world):
        counts, rows = res[dst]
        assert counts == [(s + 1) * (dst + 1) for s in range(world)]
        # segments in source order, rows in send order
        want = [[s, dst, k] for s in range(world) for k in range((s + 1) * (dst + 1))]
        assert rows == want


def _reduce_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from differentiable_tile_rasterizer_b200.pipeline import flat_gradient_buffers
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        N, sh_degree = 5, 3
        flat, views = flat_gradient_buffers(N, sh_degree, "cpu")
        flat.copy_(torch.arange(flat.numel(), dtype=torch.float32) * (rank + 1))
        views["sh"][2, 3] += 100.0 * rank  # writes through the views land in the flat buffer
        bench.reduce_gradients(flat, world)
        out.put((rank, flat.tolist(), {k: list(v.shape) for k, v in views.items()}))
    finally:
        dist.destroy_process_group()


def test_gradient_all_reduce_of_the_data_parallel_step_with_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_reduce_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = {r: (flat, shapes) for r, flat, shapes in (q.get(timeout=10) for _ in range(world))}
    N, K = 5, 16
    n = (11 + 3 * K) * N
    want = [float(i * 3) for i in range(n)]  # rank 0 contributes i, rank 1 contributes 2 i
    want[3 * N + 3 * N + 4 * N + N + 2 * N + 3] += 100.0
    for r in range(world):
        flat, shapes = res[r]
        assert flat == want
        assert shapes == {"means": [3, N], "log_scales": [3, N], "quats": [4, N], "opacity_logits": [N],
                          "sh": [3 * K, N]}
