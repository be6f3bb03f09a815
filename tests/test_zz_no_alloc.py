"""gs_cull_noalloc against gs_cull, through the C ABI.

Some users of this library cannot allocate device memory: a plugin running
inside a host application that does not own the device allocator, or a
real-time loop that may not call cudaMalloc because it synchronises the whole
device. gs_cull_noalloc serves them by keeping the cull's scratch in a static
array inside the library. This test checks that it reproduces gs_cull
exactly -- masks, active lists and counts are integer results, compared bit
for bit as everywhere else in the suite -- on two calls in a row with
different sizes and gates, which also shows that each call clears the shared
scratch it relies on. It also checks the promise itself (free device memory
is unchanged across calls on a non-default stream) and that a context the
host application created on its own gets its own copy of the scratch, whose
address the library looks up separately. It runs last (file name) and passes
both on its own in a fresh process and after the rest of the suite.
"""

import ctypes

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


def test_noalloc_cull_allocates_nothing_on_a_side_stream():
    rng = np.random.default_rng(12)
    cam = gs.camera(simple_camera(128, 96, 100.0))
    cam.campos[:] = [1.0, 2.0, -3.0]
    N = 400_000
    means = torch.from_numpy(rng.uniform(-150, 150, (3, N)).astype(np.float32)).cuda()
    imp = torch.from_numpy(rng.exponential(1.0, N).astype(np.float32)).cuda()
    side = torch.cuda.Stream()
    outs = [(torch.empty(N, dtype=torch.uint8, device="cuda"), torch.empty(N, dtype=torch.int32, device="cuda"),
             torch.empty(1, dtype=torch.int32, device="cuda")) for _ in range(3)]
    torch.cuda.synchronize()
    gs.gs_cull_noalloc(means, imp, N, cam, 120.0, 0.4, *outs[0], stream=side)  # warm-up (module load)
    side.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for k in range(3):
        gs.gs_cull_noalloc(means, imp, N, cam, 120.0 - 10 * k, 0.4, *outs[k], stream=side)
    side.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    # the last call against gs_cull on the same side stream
    ws = torch.empty(gs.gs_cull_workspace(N, cam), dtype=torch.uint8, device="cuda")
    m = torch.empty(N, dtype=torch.uint8, device="cuda")
    a = torch.empty(N, dtype=torch.int32, device="cuda")
    n = torch.empty(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    gs.gs_cull(means, imp, N, cam, 100.0, 0.4, m, a, n, ws, stream=side)
    side.synchronize()
    na = int(n.item())
    assert 0 < na < N and int(outs[2][2].item()) == na
    assert torch.equal(outs[2][0], m) and torch.equal(outs[2][1][:na], a[:na])


class _Driver:
    """The few CUDA driver calls the second-context test makes itself."""

    def __init__(self):
        self.cu = ctypes.CDLL("libcuda.so.1")

    def __call__(self, name, *args):
        rc = getattr(self.cu, name)(*args)
        assert rc == 0, f"{name} returned {rc}"


def test_noalloc_cull_in_a_context_the_application_created():
    rng = np.random.default_rng(13)
    cam = gs.camera(simple_camera(128, 96, 100.0))
    cam.campos[:] = [-2.0, 5.0, 1.0]
    N = 300_000
    means_h = np.ascontiguousarray(rng.uniform(-150, 150, (3, N)).astype(np.float32))
    imp_h = np.ascontiguousarray(rng.exponential(1.0, N).astype(np.float32))
    lod, q = 140.0, 0.35
    # in torch's (primary) context first, so the library has cached that
    # context's scratch address before the second context exists
    means, imp = torch.from_numpy(means_h).cuda(), torch.from_numpy(imp_h).cuda()
    na_primary = _cull_both(means, imp, N, cam, lod, q)
    torch.cuda.synchronize()

    cu = _Driver()
    L = gs.load()
    dev = ctypes.c_int(0)
    cu("cuDeviceGet", ctypes.byref(dev), torch.cuda.current_device())
    ctx = ctypes.c_void_p()
    cu("cuCtxCreate_v2", ctypes.byref(ctx), 0, dev)  # made current on this thread
    ptrs = []
    try:
        def alloc(nbytes):
            p = ctypes.c_uint64()
            cu("cuMemAlloc_v2", ctypes.byref(p), ctypes.c_size_t(max(nbytes, 1)))
            ptrs.append(p)
            return ctypes.c_void_p(p.value)

        d_means, d_imp = alloc(means_h.nbytes), alloc(imp_h.nbytes)
        cu("cuMemcpyHtoD_v2", ctypes.c_uint64(d_means.value), means_h.ctypes.data_as(ctypes.c_void_p),
           ctypes.c_size_t(means_h.nbytes))
        cu("cuMemcpyHtoD_v2", ctypes.c_uint64(d_imp.value), imp_h.ctypes.data_as(ctypes.c_void_p),
           ctypes.c_size_t(imp_h.nbytes))
        nbytes = ctypes.c_size_t(0)
        assert L.gs_cull(None, None, N, ctypes.byref(cam), 0.0, 0.0, None, None, None, None,
                         ctypes.byref(nbytes), None) == gs.GS_OK
        ws = alloc(nbytes.value)
        res = {}
        for which in ("workspace", "noalloc"):
            mask, act, n = alloc(N), alloc(4 * N), alloc(4)
            if which == "workspace":
                st = L.gs_cull(d_means, d_imp, N, ctypes.byref(cam), lod, q, mask, act, n, ws,
                               ctypes.byref(nbytes), None)
            else:
                st = L.gs_cull_noalloc(d_means, d_imp, N, ctypes.byref(cam), lod, q, mask, act, n, None)
            assert st == gs.GS_OK, (which, st)
            cu("cuCtxSynchronize")
            out = (np.empty(N, np.uint8), np.empty(N, np.int32), np.empty(1, np.int32))
            for h, d in zip(out, (mask, act, n)):
                cu("cuMemcpyDtoH_v2", h.ctypes.data_as(ctypes.c_void_p), ctypes.c_uint64(d.value),
                   ctypes.c_size_t(h.nbytes))
            res[which] = out
        na = int(res["workspace"][2][0])
        assert na == na_primary and int(res["noalloc"][2][0]) == na
        assert np.array_equal(res["workspace"][0], res["noalloc"][0])
        assert np.array_equal(res["workspace"][1][:na], res["noalloc"][1][:na])
    finally:
        for p in ptrs:
            cu("cuMemFree_v2", ctypes.c_uint64(p.value))
        popped = ctypes.c_void_p()
        cu("cuCtxPopCurrent_v2", ctypes.byref(popped))
        cu("cuCtxDestroy_v2", ctx)
    # and again in torch's context, after the other one is gone
    assert _cull_both(means, imp, N, cam, lod, q) == na_primary
