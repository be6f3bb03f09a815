"""gs_cull_noalloc against gs_cull, through the C ABI.

Some users of this library cannot allocate device memory: a plugin running
inside a host application that does not own the device allocator, or a
real-time loop that may not call cudaMalloc because it synchronises the whole
device. gs_cull_noalloc serves them by keeping the cull's scratch in a static
array inside the library. This test checks that it reproduces gs_cull
exactly -- masks, active lists and counts are integer results, compared bit
for bit as everywhere else in the suite -- on two calls in a row with
different sizes and gates, which also shows that each call clears the shared
scratch it relies on. It runs last (file name) and passes both on its own in
a fresh process and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

from differentiable_tile_rasterizer_b200 import gs
from tests._helpers import simple_camera

pytestmark = pytest.mark.gpu


def _cull_both(means, imp, N, cam, lod, q):
    dev = "cuda"
    ws = torch.empty(gs.gs_cull_workspace(N, cam), dtype=torch.uint8, device=dev)
    m_a = torch.full((N,), 7, dtype=torch.uint8, device=dev)
    a_a = torch.full((N,), -1, dtype=torch.int32, device=dev)
    n_a = torch.full((1,), -1, dtype=torch.int32, device=dev)
    gs.gs_cull(means, imp, N, cam, lod, q, m_a, a_a, n_a, ws)
    m_b = torch.full((N,), 7, dtype=torch.uint8, device=dev)
    a_b = torch.full((N,), -1, dtype=torch.int32, device=dev)
    n_b = torch.full((1,), -1, dtype=torch.int32, device=dev)
    gs.gs_cull_noalloc(means, imp, N, cam, lod, q, m_b, a_b, n_b)
    torch.cuda.synchronize()
    na = int(n_a.item())
    assert int(n_b.item()) == na
    assert torch.equal(m_a, m_b)
    assert torch.equal(a_a[:na], a_b[:na])
    return na


def test_noalloc_cull_matches_workspace_cull_on_two_calls():
    rng = np.random.default_rng(11)
    cam = gs.camera(simple_camera(128, 96, 100.0))
    cam.campos[:] = [4.0, -3.0, 2.0]
    results = []
    # two calls in a row with different sizes, gates and quantiles
    for N, lod, q in [(1_000_000, 150.0, 0.3), (250_000, 0.0, 0.55)]:
        means = torch.from_numpy(rng.uniform(-200, 200, (3, N)).astype(np.float32)).cuda()
        imp = torch.from_numpy(rng.exponential(1.0, N).astype(np.float32)).cuda()
        na = _cull_both(means, imp, N, cam, lod, q)
        assert 0 < na < N
        results.append(na)
    assert results[0] != results[1]


def test_noalloc_cull_rejects_sizes_beyond_its_static_scratch():
    cam = gs.camera(simple_camera(64, 64, 50.0))
    with pytest.raises(gs.GsError) as ei:
        gs.gs_cull_noalloc(None, None, gs.GS_CULL_NOALLOC_MAX_N + 1, cam, 0.0, 0.0, None, None, None)
    assert ei.value.status == gs.GS_ERR_INVALID_ARGUMENT
