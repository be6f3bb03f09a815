"""The rasterizer's public Python API: one view forward and backward through
the C entry points (gs_cull, gs_preprocess, gs_bin_sort(_async),
gs_tile_order, gs_rasterize_fwd, gs_rasterize_bwd), plus the multi-view
renderer and the quantised SH optimizer. Torch only allocates device memory
and supplies the stream; every stage runs in libgs.so.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from . import gs


@dataclasses.dataclass
class GaussianParams:
    """Device-resident parameters in the library's SoA layout."""
    means: torch.Tensor        # [3][N]
    log_scales: torch.Tensor   # [3][N]
    quats: torch.Tensor        # [4][N]
    opacity_logits: torch.Tensor  # [N]
    sh: torch.Tensor           # [K*3][N]
    sh_degree: int
    importance: Optional[torch.Tensor] = None  # [N]

    @property
    def N(self) -> int:
        return int(self.opacity_logits.shape[0])

    @property
    def K(self) -> int:
        return (self.sh_degree + 1) ** 2

    @staticmethod
    def from_scene(scene, device="cuda") -> "GaussianParams":
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        return GaussianParams(t(scene.means), t(scene.log_scales), t(scene.quats),
                              t(scene.opacity_logits), t(scene.sh), scene.sh_degree,
                              None if scene.importance is None else t(scene.importance))

    @staticmethod
    def empty_like_host(scene, pin=True):
        """Pinned host copies of a scene's parameters (for host-buffer calls)."""
        f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory() if pin else torch.from_numpy(a)
        return {k: f(getattr(scene, k)) for k in ("means", "log_scales", "quats", "opacity_logits", "sh")}


class _Stage:
    """One stage of a view: an NVTX range named gs.<stage> (visible to
    profilers that record NVTX) and, when a store is given, CUDA events
    around the stage's launches."""

    def __init__(self, name, store=None):
        self.name, self.store = name, store

    def __enter__(self):
        torch.cuda.nvtx.range_push("gs." + self.name)
        if self.store is not None:
            self.start = torch.cuda.Event(enable_timing=True)
            self.end = torch.cuda.Event(enable_timing=True)
            self.start.record()
        return self

    def __exit__(self, *a):
        if self.store is not None:
            self.end.record()
            self.store.append((self.start, self.end))
        torch.cuda.nvtx.range_pop()
        return False


def _u8(n, dev):
    return torch.empty(max(int(n), 1), dtype=torch.uint8, device=dev)


class Rasterizer:
    """Buffers and calls for rendering one view of N Gaussians at W x H.

    forward() runs cull (when a gate is on) -> preprocess -> bin_sort ->
    tile_order -> rasterize_fwd and keeps what backward() needs (including
    the forward's hit bytes); backward() runs rasterize_bwd. Buffers are
    allocated once (the instance capacity grows when gs_bin_sort reports it
    is too small) and reused across calls. In deferred mode no call reads
    the device from the host, so a whole step can be captured in a CUDA
    graph.
    """

    def __init__(self, N: int, sh_degree: int, width: int, height: int, device=None,
                 capacity: Optional[int] = None):
        self.dev = torch.device(device or "cuda")
        self.N, self.sh_degree, self.W, self.H = int(N), int(sh_degree), int(width), int(height)
        self.K = (sh_degree + 1) ** 2
        self.TW, self.TH = (width + 15) // 16, (height + 15) // 16
        self.TT = self.TW * self.TH
        n, d = max(self.N, 1), self.dev
        f32 = dict(dtype=torch.float32, device=d)
        i32 = dict(dtype=torch.int32, device=d)
        self.rec = {"xyzo": torch.empty((n, 4), **f32), "conic": torch.empty((n, 4), **f32),
                    "rgb": torch.empty((n, 4), **f32), "radius": torch.empty(n, **i32),
                    "rect": torch.empty((n, 4), dtype=torch.int16, device=d),
                    "tiles": torch.empty(n, **i32)}
        self.offsets = torch.empty(n, **i32)
        self.mask = torch.empty(n, dtype=torch.uint8, device=d)
        self.active_idx = torch.empty(n, **i32)
        self.n_active = torch.zeros(1, **i32)
        self.image = torch.empty((3, height, width), **f32)
        self.final_T = torch.empty((height, width), **f32)
        self.n_contrib = torch.empty((height, width), **i32)
        self.last = torch.empty((height, width), **i32)
        self.ranges = torch.empty((self.TT, 2), **i32)
        # Tiles longest list first (gs_tile_order), computed after every bin
        # sort and given to the raster launches; None: CTA b takes tile b.
        self.schedule_tiles = True
        self.tile_order = torch.arange(max(self.TT, 1), **i32)
        # The forward writes one byte per list entry with the 8x4 pixel
        # blocks where it blended, and the backward walks only those
        # (gs_rasterize_fwd's hit_bits). False: the backward tests every
        # entry's blend region itself.
        self.use_hit_bits = True
        self._hits_fresh = False  # hit_bits hold the current lists' bytes
        self.grad2d = torch.empty((n, 12), **f32)
        self.grads = {"means": torch.empty((3, n), **f32), "log_scales": torch.empty((3, n), **f32),
                      "quats": torch.empty((4, n), **f32), "opacity_logits": torch.empty(n, **f32),
                      "sh": torch.empty((3 * self.K, n), **f32)}
        self._proj = gs.projected(self.rec)
        self.capacity = 0
        self.keys = self.vals = self.sort_ws = None
        self._cam_wh = None
        self._ensure_capacity(capacity if capacity is not None else max(4 * self.N, 1024))
        cam_probe = gs.GsCamera()
        cam_probe.width, cam_probe.height = width, height
        self.cull_ws = _u8(gs.gs_cull_workspace(self.N, cam_probe), d)
        self.n_instances = 0
        self.params = None
        self.cam = None
        self.bg = (0.0, 0.0, 0.0)
        self.culled = False
        # Optional per-stage CUDA-event timing: {stage: [(start, end), ...]}.
        self.stage_events = None
        # Also produce the record-order scan of tiles_touched (gs_bin_sort offsets).
        self.want_offsets = False
        # Deferred checking: forward() enqueues the bin/sort without a host
        # round trip (gs_bin_sort_async); each view's (instances, status) stays
        # in a device slot until check() reads them all at once.
        self.deferred = False
        self._results = torch.zeros((4096, 2), dtype=torch.int64, device=d)
        self._n_pending = 0

    def _timed(self, stage):
        ev = self.stage_events
        return _Stage(stage, None if ev is None else ev.setdefault(stage, []))

    def _ensure_capacity(self, cap: int):
        if cap <= self.capacity:
            return
        cap = int(cap)
        self.keys = torch.empty(max(cap, 1), dtype=torch.int64, device=self.dev)
        self.vals = torch.empty(max(cap, 1), dtype=torch.int32, device=self.dev)
        self.hit_bits = torch.empty((max(cap, 1) + 3) // 4 * 4, dtype=torch.uint8, device=self.dev)
        probe = gs.GsCamera()
        probe.width, probe.height = self.W, self.H
        self.sort_ws = _u8(gs.gs_bin_sort_workspace(self.N, probe, cap), self.dev)
        self.capacity = cap

    # ------------------------------------------------------------------ stages
    def cull(self, params: GaussianParams, cam: gs.GsCamera, lod_dist=0.0, importance_q=0.0):
        with self._timed("cull"):
            gs.gs_cull(params.means, params.importance if importance_q > 0 else None, self.N, cam,
                       lod_dist, importance_q, self.mask, self.active_idx, self.n_active, self.cull_ws)
        self.culled = True

    def _gate(self, params: GaussianParams, cam: gs.GsCamera, lod_dist, importance_q):
        """The cull of forward(): with both gates off every Gaussian is active
        and its active list would be the identity, so the records are
        indexed by Gaussian directly and no cull runs."""
        if lod_dist > 0 or importance_q > 0:
            self.cull(params, cam, lod_dist, importance_q)
        else:
            self.culled = False

    def preprocess(self, params: GaussianParams, cam: gs.GsCamera):
        act = self.active_idx if self.culled else None
        na = self.n_active if self.culled else None
        with self._timed("preprocess"):
            gs.gs_preprocess(params.means, params.log_scales, params.quats, params.opacity_logits,
                             params.sh, params.sh_degree, self.N, act, na, cam, self._proj)

    def bin_sort(self, cam: gs.GsCamera) -> int:
        with self._timed("bin_sort"):
            return self._bin_sort(cam)

    def _order(self):
        return self.tile_order if self.schedule_tiles else None

    def _hits(self):
        """hit_bits for a forward (which writes them)."""
        if not self.use_hit_bits:
            return None
        self._hits_fresh = True
        return self.hit_bits

    def _hits_in(self):
        """hit_bits for a backward: only when a forward wrote them for the
        current lists."""
        return self.hit_bits if self.use_hit_bits and self._hits_fresh else None

    def _bin_sort(self, cam: gs.GsCamera):
        offs = self.offsets if self.want_offsets else None
        self._hits_fresh = False
        if self.deferred:
            if self._n_pending == self._results.shape[0]:
                self.check()
            gs.gs_bin_sort_async(self._proj, self.N, cam, offs, self.keys, self.vals, self.capacity,
                                 self.ranges, self._results[self._n_pending], self.sort_ws)
            self._n_pending += 1
            if self.schedule_tiles:
                gs.gs_tile_order(self.ranges, self.TT, self.tile_order)
            return None
        st, ni = gs.gs_bin_sort(self._proj, self.N, cam, offs, self.keys, self.vals, self.capacity,
                                self.ranges, self.sort_ws, raise_on_capacity=False)
        if st == gs.GS_ERR_CAPACITY:
            self._ensure_capacity(int(ni * 1.25) + 1024)
            st, ni = gs.gs_bin_sort(self._proj, self.N, cam, offs, self.keys, self.vals,
                                    self.capacity, self.ranges, self.sort_ws)
        self.n_instances = ni
        if self.schedule_tiles:
            gs.gs_tile_order(self.ranges, self.TT, self.tile_order)
        return ni

    def forward_importance(self, params: GaussianParams, cam, importance: torch.Tensor, bg=(0.0, 0.0, 0.0),
                           lod_dist=0.0, importance_q=0.0) -> torch.Tensor:
        """The forward of one view that also adds each Gaussian's importance
        weight (sum over the view's pixels of alpha * T) to `importance`
        (float32 [N] on the device; zero it once, call once per view)."""
        c = cam if isinstance(cam, gs.GsCamera) else gs.camera(cam)
        if (c.width, c.height) != (self.W, self.H):
            raise ValueError("camera size differs from the rasterizer's")
        if importance.dtype != torch.float32 or importance.numel() != self.N or not importance.is_cuda:
            raise ValueError("importance must be a float32 CUDA tensor of N elements")
        self.params, self.cam, self.bg = params, c, tuple(float(b) for b in bg)
        self._gate(params, c, lod_dist, importance_q)
        self.preprocess(params, c)
        self.bin_sort(c)
        with self._timed("raster_fwd_importance"):
            gs.gs_rasterize_fwd_importance(self._proj, self.vals, self.ranges, c, self.bg,
                                           self.active_idx if self.culled else None,
                                           self.image, self.final_T, self.n_contrib, self.last, importance,
                                           tile_order=self._order(), hit_bits=self._hits())
        return self.image

    def accumulate_grad_stats(self, norm_sum: torch.Tensor, view_count: torch.Tensor):
        """After backward(): adds this view's |dL/d(mean2D)| of every visible
        Gaussian to norm_sum (float32 [N]) and 1 to view_count (int32 [N])."""
        act = self.active_idx if self.culled else None
        na = self.n_active if self.culled else None
        gs.gs_accumulate_grad2d_norm(self.grad2d, self.rec["tiles"], act, na, self.N, norm_sum, view_count)

    def check(self) -> list:
        """Instance counts of the views binned in deferred mode since the last
        check (one host read). Raises GsError if one of them failed; after a
        capacity failure the buffers have been grown, so repeating those views
        succeeds."""
        k = self._n_pending
        self._n_pending = 0
        if k == 0:
            return []
        res = self._results[:k].cpu().tolist()
        counts = [int(ni) for ni, _ in res]
        self.n_instances = counts[-1]
        for ni, st in res:
            if st == gs.GS_ERR_CAPACITY:
                self._ensure_capacity(int(max(counts) * 1.25) + 1024)
            if st != gs.GS_OK:
                gs._check("gs_bin_sort_async", int(st))
        return counts

    def raster_fwd(self, cam: gs.GsCamera, bg):
        with self._timed("raster_fwd"):
            gs.gs_rasterize_fwd(self._proj, self.vals, self.ranges, cam, bg, self.image, self.final_T,
                                self.n_contrib, self.last, tile_order=self._order(), hit_bits=self._hits())

    # ------------------------------------------------------------------ public
    def forward(self, params: GaussianParams, cam, bg=(0.0, 0.0, 0.0), lod_dist=0.0,
                importance_q=0.0) -> torch.Tensor:
        c = cam if isinstance(cam, gs.GsCamera) else gs.camera(cam)
        if (c.width, c.height) != (self.W, self.H):
            raise ValueError("camera size differs from the rasterizer's")
        self.params, self.cam, self.bg = params, c, tuple(float(b) for b in bg)
        self._gate(params, c, lod_dist, importance_q)
        self.preprocess(params, c)
        self.bin_sort(c)
        self.raster_fwd(c, self.bg)
        return self.image

    def backward(self, dL_dimage: torch.Tensor, accumulate_into: Optional[dict] = None) -> dict:
        """Gradients of the last forward's view. Into self.grads (overwritten)
        or, with accumulate_into (a dict of parameter-shaped float32 tensors,
        zeroed by the caller before the first view), added to those: the
        gradient of a loss summed over views. Accumulating calls on the same
        tensors must run in order on one stream."""
        p, c = self.params, self.cam
        act = self.active_idx if self.culled else None
        na = self.n_active if self.culled else None
        mask = self.mask if self.culled else None
        g = self.grads
        if accumulate_into is not None:
            a = accumulate_into
            with self._timed("raster_bwd"):
                gs.gs_rasterize_bwd_2d(self._proj, self.N, self.vals, self.ranges, c, self.bg, self.final_T,
                                       self.last, dL_dimage, self.grad2d, tile_order=self._order(),
                                       hit_bits=self._hits_in())
            with self._timed("preprocess_bwd"):
                gs.gs_preprocess_bwd_accumulate(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh,
                                                p.sh_degree, self.N, act, na, c, self._proj, self.grad2d,
                                                a["means"], a["log_scales"], a["quats"], a["opacity_logits"],
                                                a["sh"])
            return a
        if self.stage_events is None:
            with _Stage("backward"):
                gs.gs_rasterize_bwd(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh, p.sh_degree,
                                    self.N, act, na, mask, c, self._proj, self.vals, self.ranges, self.bg,
                                    self.final_T, self.last, dL_dimage, self.grad2d, g["means"],
                                    g["log_scales"], g["quats"], g["opacity_logits"], g["sh"],
                                    tile_order=self._order(), hit_bits=self._hits_in())
            return g
        # the same two parts as separate calls, so each can be timed
        with self._timed("raster_bwd"):
            gs.gs_rasterize_bwd_2d(self._proj, self.N, self.vals, self.ranges, c, self.bg, self.final_T,
                                   self.last, dL_dimage, self.grad2d, tile_order=self._order(),
                                   hit_bits=self._hits_in())
        with self._timed("preprocess_bwd"):
            gs.gs_preprocess_bwd(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh, p.sh_degree,
                                 self.N, act, na, mask, c, self._proj, self.grad2d, g["means"],
                                 g["log_scales"], g["quats"], g["opacity_logits"], g["sh"])
        return g

    def backward_2d(self, dL_dimage: torch.Tensor):
        """Part 1 of backward(): the per-record 2-D gradients (self.grad2d)."""
        with self._timed("raster_bwd"):
            gs.gs_rasterize_bwd_2d(self._proj, self.N, self.vals, self.ranges, self.cam, self.bg, self.final_T,
                                   self.last, dL_dimage, self.grad2d, tile_order=self._order(),
                                   hit_bits=self._hits_in())

    def backward_params(self, into: dict, accumulate: bool):
        """Part 2 of backward(): parameter gradients from self.grad2d, written
        into `into` (a dict of parameter-shaped float32 tensors), or added to
        it when accumulate is set."""
        p, c = self.params, self.cam
        act = self.active_idx if self.culled else None
        na = self.n_active if self.culled else None
        with self._timed("preprocess_bwd"):
            if accumulate:
                gs.gs_preprocess_bwd_accumulate(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh,
                                                p.sh_degree, self.N, act, na, c, self._proj, self.grad2d,
                                                into["means"], into["log_scales"], into["quats"],
                                                into["opacity_logits"], into["sh"])
            else:
                gs.gs_preprocess_bwd(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh, p.sh_degree,
                                     self.N, act, na, self.mask if self.culled else None, c, self._proj,
                                     self.grad2d, into["means"], into["log_scales"], into["quats"],
                                     into["opacity_logits"], into["sh"])

    def work_counts(self) -> dict:
        """Per-view work of the last forward (device reductions, then one sync):
        active Gaussians A (N without a cull), visible Gaussians V, instances
        I, forward-evaluated pairs E (pairs of a
        pixel and an entry of its tile's list up to the pixel's stop), backward
        pairs E_bwd (entries before each pixel's last blend) and blends B."""
        H, W = self.H, self.W
        lens = (self.ranges[:, 1] - self.ranges[:, 0]).to(torch.int64)
        ty = torch.arange(H, device=self.dev) // 16
        tx = torch.arange(W, device=self.dev) // 16
        tile = (ty[:, None] * self.TW + tx[None, :]).reshape(-1)
        plen = lens[tile].reshape(H, W)
        last = self.last.to(torch.int64)
        stopped = self.final_T < 1e-4
        E = torch.where(stopped, last, plen).sum()
        A = self.n_active[0].to(torch.int64) if self.culled else torch.tensor(self.N, device=self.dev)
        out = torch.stack([(self.rec["tiles"] > 0).sum().to(torch.int64), E, last.sum(),
                           self.n_contrib.to(torch.int64).sum(), A]).cpu().tolist()
        return {"V": out[0], "I": self.n_instances, "E": out[1], "E_bwd": out[2], "B": out[3], "A": out[4],
                "culled": self.culled}

    def records_numpy(self) -> dict:
        r = {k: v.cpu().numpy() for k, v in self.rec.items()}
        r["rect"] = r["rect"].view(np.uint16)
        return r

    def bins_numpy(self) -> dict:
        I = self.n_instances
        return {"keys": self.keys[:I].cpu().numpy().view(np.uint64),
                "vals": self.vals[:I].cpu().numpy().view(np.uint32),
                "ranges": self.ranges.cpu().numpy().view(np.uint32),
                "offsets": self.offsets.cpu().numpy(), "n_instances": I}


def flat_gradient_buffers(N: int, sh_degree: int, device):
    """One flat float32 buffer for a whole parameter gradient and a dict of
    views of it in the library's SoA shapes (means [3][N], log_scales
    [3][N], quats [4][N], opacity_logits [N], sh [3K][N])."""
    K, n = (sh_degree + 1) ** 2, max(int(N), 1)
    flat = torch.empty((11 + 3 * K) * n, dtype=torch.float32, device=device)
    views, o = {}, 0
    for name, rows in (("means", 3), ("log_scales", 3), ("quats", 4), ("opacity_logits", 1), ("sh", 3 * K)):
        v = flat[o: o + rows * n]
        views[name] = v if name == "opacity_logits" else v.view(rows, n)
        o += rows * n
    return flat, views


class MultiViewRenderer:
    """Rendering of several views of one model: one pass over the
    parameters projects every Gaussian into all views
    (gs_preprocess_multiview), then each view runs its bin/sort and raster
    forward on its own buffers (a Rasterizer per view). No cull: every
    Gaussian is projected into every view. backward() gives the parameter
    gradients of a loss summed over the views, again with one pass over the
    parameters (gs_preprocess_bwd_multiview).

    The views' bin/sorts, raster forwards and raster backwards run on
    n_streams streams (view v on stream v mod n_streams), forked from and
    joined to the caller's stream, so that the views' latency-bound sort
    kernels run beside one another (and beside other views' raster kernels
    where the SMs have room). With deferred mode on (set_deferred) no call
    waits on the host; otherwise each bin/sort waits for its own stream only.
    While stage timing is on (stage_events not None) the views run one after
    another on one stream, so that each stage's events bracket its own work."""

    def __init__(self, N: int, sh_degree: int, cams, device=None, capacity: Optional[int] = None,
                 n_streams: int = 4):
        self.cams = [c if isinstance(c, gs.GsCamera) else gs.camera(c) for c in cams]
        if not 0 < len(self.cams) <= gs.GS_MAX_VIEWS:
            raise ValueError(f"1 .. {gs.GS_MAX_VIEWS} views per pass")
        self.N, self.sh_degree = int(N), int(sh_degree)
        self.views = [Rasterizer(N, sh_degree, c.width, c.height, device=device, capacity=capacity)
                      for c in self.cams]
        d = torch.device(device or "cuda")
        self.streams = [torch.cuda.Stream(device=d) for _ in range(min(max(int(n_streams), 1), len(self.cams)))]
        self.stage_events = None
        self.params = None
        # parameter gradients of the loss summed over the views (backward):
        # views into one flat buffer, so that one collective can reduce them
        self.grads_flat, self.grads = flat_gradient_buffers(self.N, self.sh_degree, d)

    def _timed(self, stage):
        ev = self.stage_events
        return _Stage(stage, None if ev is None else ev.setdefault(stage, []))

    def forward(self, params: GaussianParams, bg=(0.0, 0.0, 0.0)) -> list:
        bg = tuple(float(b) for b in bg)
        self.params = params
        with self._timed("preprocess_multiview"):
            gs.gs_preprocess_multiview(params.means, params.log_scales, params.quats, params.opacity_logits,
                                       params.sh, params.sh_degree, self.N, self.cams,
                                       [R._proj for R in self.views])
        cur = torch.cuda.current_stream()
        streams = self.streams if self.stage_events is None else self.streams[:1]
        for st in streams:
            st.wait_stream(cur)
        for v, (R, c) in enumerate(zip(self.views, self.cams)):
            R.params, R.cam, R.bg, R.culled = params, c, bg, False
            with torch.cuda.stream(streams[v % len(streams)]):
                with self._timed("bin_sort"):
                    R._bin_sort(c)
                with self._timed("raster_fwd"):
                    gs.gs_rasterize_fwd(R._proj, R.vals, R.ranges, c, bg, R.image, R.final_T, R.n_contrib,
                                        R.last, tile_order=R._order(), hit_bits=R._hits())
        for st in streams:
            cur.wait_stream(st)
        return [R.image for R in self.views]

    def backward(self, dL_dimages, into: Optional[dict] = None) -> dict:
        """Parameter gradients of a loss summed over the views of the last
        forward, given each view's dL/dimage ([3][H][W] float32 on the
        device): per view the 2-D gradients (gs_rasterize_bwd_2d, on the
        views' streams, with the forward's hit bytes), then one pass over
        the parameters that chains and sums them
        (gs_preprocess_bwd_multiview). Written into `into` (a dict of
        parameter-shaped float32 tensors) if given, else into self.grads;
        returns that dict (every row overwritten)."""
        if len(dL_dimages) != len(self.views):
            raise ValueError("one image gradient per view")
        p = self.params
        if p is None:
            raise RuntimeError("backward() before forward()")
        cur = torch.cuda.current_stream()
        streams = self.streams if self.stage_events is None else self.streams[:1]
        for st in streams:
            st.wait_stream(cur)
        for v, (R, g) in enumerate(zip(self.views, dL_dimages)):
            with torch.cuda.stream(streams[v % len(streams)]):
                with self._timed("raster_bwd"):
                    gs.gs_rasterize_bwd_2d(R._proj, R.N, R.vals, R.ranges, R.cam, R.bg, R.final_T, R.last, g,
                                           R.grad2d, tile_order=R._order(), hit_bits=R._hits_in())
        for st in streams:
            cur.wait_stream(st)
        a = self.grads if into is None else into
        with self._timed("preprocess_bwd_multiview"):
            gs.gs_preprocess_bwd_multiview(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh, p.sh_degree,
                                           self.N, self.cams, [R._proj for R in self.views],
                                           [R.grad2d for R in self.views], a["means"], a["log_scales"],
                                           a["quats"], a["opacity_logits"], a["sh"])
        return a

    def set_deferred(self, on: bool):
        for R in self.views:
            R.deferred = on

    def check(self) -> list:
        return [R.check() for R in self.views]


class QuantizedSHAdam:
    """Adam over the view-dependent SH coefficients kept as 16-bit block codes,
    with both moments as 8-bit block codes of their logarithms
    (gs_adam_sh_quant). Planes 3 .. 3K - 1 of the SH parameters (the DC plane
    stays in fp32); 256 consecutive Gaussians of a plane share a (lo, hi)."""

    def __init__(self, N: int, sh_degree: int, lr=2.5e-3 / 20.0, beta1=0.9, beta2=0.999, eps=1e-15,
                 code_scale=1e-15, device=None):
        if sh_degree < 1:
            raise ValueError("no view-dependent SH coefficients at degree 0")
        d = torch.device(device or "cuda")
        self.N, self.K = int(N), (sh_degree + 1) ** 2
        self.U = 3 * (self.K - 1)
        self.nblk = (self.N + 255) // 256
        pad = self.nblk * 256
        self.pc = torch.zeros((self.U, pad), dtype=torch.int16, device=d)  # uint16 codes
        self.mc = torch.zeros((self.U, pad), dtype=torch.uint8, device=d)
        self.vc = torch.zeros((self.U, pad), dtype=torch.uint8, device=d)
        self.pb = torch.zeros((self.U, self.nblk, 2), dtype=torch.float32, device=d)
        self.mb = torch.zeros_like(self.pb)
        self.vb = torch.zeros_like(self.pb)
        self.lr, self.beta1, self.beta2, self.eps, self.code_scale = lr, beta1, beta2, eps, code_scale
        self.step_count = 0

    def load(self, sh: torch.Tensor):
        """Codes of the SH planes 3.. of sh [3K][N] (moments reset to zero)."""
        gs.gs_quant_encode(sh[3:], self.U, self.N, 16, self.pc, self.pb)
        for t in (self.mc, self.vc, self.mb, self.vb):
            t.zero_()
        self.step_count = 0

    def step(self, d_sh: torch.Tensor):
        """One Adam step from the gradients d_sh [3K][N] (planes 3.. are used)."""
        self.step_count += 1
        gs.gs_adam_sh_quant(d_sh[3:], self.U, self.N, self.pc, self.pb, self.mc, self.mb, self.vc, self.vb,
                            self.lr, self.beta1, self.beta2, self.eps, self.code_scale, self.step_count)

    def store(self, sh: torch.Tensor):
        """Decoded values into the SH planes 3.. of sh [3K][N] (for rendering)."""
        gs.gs_quant_decode(self.pc, self.pb, self.U, self.N, 16, sh[3:])
