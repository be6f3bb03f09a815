"""Index-interleaved multi-GPU rendering with one exchange of projected
records (BlitzGS write-up, section 2.1): rank r of G holds Gaussians
r, r + G, r + 2G, ... and owns a band of tile rows; every rank projects its
own Gaussians, one all-to-all routes each projected Gaussian to the ranks
whose bands it touches, and each rank bins, sorts and rasterises its band.
The backward runs on the band and one reverse all-to-all returns the 2-D
gradients to the ranks that own the Gaussians.

InterleavedRank holds one rank's buffers and splits its work into phases
around the two exchanges, so the same code runs with a torch.distributed
group (`DistExchange`: NCCL between GPUs, gloo on CPU tensors) or with all
ranks emulated in one process on one GPU (`emulate`). Every computing step
is a libgs call; this module only sizes buffers and moves them between the
calls.
"""

from typing import List, Optional, Sequence

import numpy as np
import torch

from . import gs
from .pipeline import GaussianParams, Rasterizer

WIRE = gs.GS_WIRE_RECORD_BYTES


def band_rows(rank: int, world: int, tiles_y: int):
    """Tile rows [lo, hi) owned by `rank` with equal bands."""
    return rank * tiles_y // world, (rank + 1) * tiles_y // world


def equal_bands(world: int, tiles_y: int) -> List[int]:
    """First tile row of every rank's band, and tiles_y: equal row counts."""
    return [q * tiles_y // world for q in range(world + 1)]


def balance_bands(row_cost: Sequence[float], world: int) -> List[int]:
    """Band starts (world + 1 values, 0 .. len(row_cost)) of contiguous row
    bands in rank order whose largest summed cost is the least any such
    partition reaches: a binary search over that largest cost, each candidate
    checked by filling rows greedily. The cost of a row is the work its
    tiles take (for instance the list entries of its tiles in a previous
    view). With no cost at all the bands are equal."""
    cost = np.asarray(row_cost, dtype=np.float64)
    TH = int(cost.size)
    if world <= 1 or TH == 0 or not (cost.sum() > 0):
        return equal_bands(world, TH)

    def cuts(limit):
        starts, acc = [0], 0.0
        for r, c in enumerate(cost):
            if acc + c > limit and acc > 0:
                starts.append(r)
                acc = 0.0
            acc += c
        return starts

    lo, hi = float(cost.max()), float(cost.sum())
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if len(cuts(mid)) <= world:
            hi = mid
        else:
            lo = mid
    starts = cuts(hi)
    while len(starts) < world:  # fewer bands were needed: split the last rows off as empty bands
        starts.append(TH)
    return starts + [TH]


def local_params(params: GaussianParams, rank: int, world: int) -> GaussianParams:
    """The Gaussians rank `rank` holds: global indices rank, rank + world, ..."""
    pick = lambda t: t[..., rank::world].contiguous()
    imp = None if params.importance is None else pick(params.importance)
    return GaussianParams(pick(params.means), pick(params.log_scales), pick(params.quats),
                          pick(params.opacity_logits), pick(params.sh), params.sh_degree, imp)


class InterleavedRank:
    def __init__(self, n_local: int, sh_degree: int, width: int, height: int, rank: int, world: int,
                 device=None, recv_capacity: Optional[int] = None, band_starts: Optional[Sequence[int]] = None):
        if not 1 <= world <= gs.GS_MAX_RANKS or not 0 <= rank < world:
            raise ValueError("bad rank / world")
        self.rank, self.world = rank, world
        self.dev = torch.device(device or "cuda")
        self.local = Rasterizer(n_local, sh_degree, width, height, device=self.dev)
        self.set_bands(band_starts if band_starts is not None else equal_bands(world, self.local.TH))
        self.sh_degree, self.W, self.H = sh_degree, width, height
        self._band_cap = 0
        self.band: Optional[Rasterizer] = None
        self._ensure_band(recv_capacity or max(2 * n_local, 1024))
        nc = int(gs.load().gs_route_ctas(max(n_local, 1)))
        self.mask = torch.empty(max(n_local, 1), dtype=torch.int32, device=self.dev)
        self.cta_counts = torch.empty(nc * world, dtype=torch.int32, device=self.dev)
        self.totals = torch.empty(world, dtype=torch.int64, device=self.dev)
        self.dst_off = torch.empty(world, dtype=torch.int64, device=self.dev)

    def set_bands(self, band_starts: Sequence[int]):
        """The tile rows every rank owns (the same list on every rank)."""
        b = [int(v) for v in band_starts]
        if len(b) != self.world + 1 or b[0] != 0 or b[-1] != self.local.TH or any(
                x > y for x, y in zip(b, b[1:])):
            raise ValueError("band starts must rise from 0 to the tile rows, one band per rank")
        self.bands = b
        self.row_lo, self.row_hi = b[self.rank], b[self.rank + 1]

    def band_row_costs(self) -> np.ndarray:
        """List entries per tile row of this rank's band in the last render
        (zero for the other rows): the work measure balance_bands takes."""
        B = self.band
        lens = (B.ranges[:, 1] - B.ranges[:, 0]).to(torch.int64).cpu().numpy().reshape(B.TH, B.TW)
        out = np.zeros(B.TH, np.float64)
        out[self.row_lo:self.row_hi] = lens[self.row_lo:self.row_hi].sum(axis=1)
        return out

    def _ensure_band(self, n: int):
        if n <= self._band_cap:
            return
        cap = int(n * 1.25) + 1024
        self.band = Rasterizer(cap, self.sh_degree, self.W, self.H, device=self.dev, capacity=8 * cap)
        self._band_cap = cap

    # ---------------------------------------------------------------- forward
    def project(self, params: GaussianParams, cam):
        """Preprocess the local Gaussians and route them to the bands: the
        records per destination (self.totals) and their first slots in the
        send buffer (self.dst_off) stay on the device."""
        c = cam if isinstance(cam, gs.GsCamera) else gs.camera(cam)
        L = self.local
        L.params, L.cam = params, c
        L.culled = False
        L.preprocess(params, c)
        gs.gs_route_count(L._proj, L.N, self.world, L.TH, self.mask, self.cta_counts, self.totals,
                          band_starts=self.bands, dst_offsets=self.dst_off)

    def pack(self, counts: List[int]) -> torch.Tensor:
        """The wire records for every rank, given this rank's send counts (the
        host copy of self.totals). Returns send bytes [sum counts * 64]."""
        L = self.local
        self.sent = int(sum(counts))
        send = torch.empty(max(self.sent, 1) * WIRE, dtype=torch.uint8, device=self.dev)
        self.src_idx = torch.empty(max(self.sent, 1), dtype=torch.int32, device=self.dev)
        gs.gs_route_pack(L._proj, self.mask, L.N, self.world, self.rank, self.cta_counts, self.dst_off, send,
                         self.src_idx)
        self.send_counts = [int(v) for v in counts]
        return send[: self.sent * WIRE]

    def project_and_pack(self, params: GaussianParams, cam, lod_dist=0.0):
        """project() and pack() with one host read of the counts. Returns
        (send bytes [sum counts * 64] uint8, counts per rank)."""
        self.project(params, cam)
        counts = [int(v) for v in self.totals.cpu().tolist()]
        return self.pack(counts), counts

    def receive_and_render(self, recv: torch.Tensor, recv_counts: List[int], cam, bg=(0.0, 0.0, 0.0)):
        """Merge the received records (one segment per source rank, in rank
        order), bin, sort and rasterise this rank's band. Returns the image;
        rows outside the band are not this rank's."""
        c = cam if isinstance(cam, gs.GsCamera) else gs.camera(cam)
        n_recv = int(sum(recv_counts))
        self._ensure_band(n_recv)
        B = self.band
        seg = [0]
        for v in recv_counts:
            seg.append(seg[-1] + int(v))
        self.recv_counts = [int(v) for v in recv_counts]
        self.n_recv = n_recv
        self.perm = torch.empty(max(n_recv, 1), dtype=torch.int32, device=self.dev)
        B.rec["tiles"][n_recv:].zero_()  # slots past the received records see no tile
        gs.gs_merge_received(recv, torch.tensor(seg, dtype=torch.int64, device=self.dev), self.world, n_recv,
                             self.row_lo, self.row_hi, B._proj, self.perm)
        B.params, B.cam, B.bg, B.culled = None, c, tuple(float(b) for b in bg), False
        B._bin_sort(c)
        B.raster_fwd(c, B.bg)
        return B.image

    # --------------------------------------------------------------- backward
    def backward_band(self, dL_dimage: torch.Tensor):
        """2-D gradients of the band's records, in received order (to be sent
        back with the received counts as the splits)."""
        B = self.band
        gs.gs_rasterize_bwd_2d(B._proj, B.N, B.vals, B.ranges, B.cam, B.bg, B.final_T, B.last, dL_dimage,
                               B.grad2d, tile_order=B._order(), hit_bits=B._hits_in())
        back = torch.empty((max(self.n_recv, 1), 12), dtype=torch.float32, device=self.dev)
        gs.gs_unmerge_grad2d(B.grad2d, self.perm, self.n_recv, back)
        return back[: self.n_recv], self.recv_counts

    def finish_backward(self, ret: torch.Tensor) -> dict:
        """Add the returned rows into the local 2-D gradients and chain them to
        the local parameters. `ret` is in send order (the reverse exchange of
        what project_and_pack sent). Returns the local parameter gradients."""
        L = self.local
        L.grad2d.zero_()
        gs.gs_return_grad2d(ret, self.src_idx, self.sent, L.grad2d)
        p, g = L.params, L.grads
        gs.gs_preprocess_bwd(p.means, p.log_scales, p.quats, p.opacity_logits, p.sh, p.sh_degree, L.N, None, None,
                             None, L.cam, L._proj, L.grad2d, g["means"], g["log_scales"], g["quats"],
                             g["opacity_logits"], g["sh"])
        return g


class DistExchange:
    """The two all-to-alls over a torch.distributed group: counts, then the
    payload (wire records forward, gradient rows backward).

    host_staging: the collectives run on host copies of the tensors (a gloo
    group, whose all-to-all takes CPU tensors) and the results are copied back
    to the device; otherwise they run on the device tensors (NCCL)."""

    def __init__(self, group=None, host_staging: bool = False):
        import torch.distributed as dist
        self.dist, self.group, self.host = dist, group, bool(host_staging)

    def counts(self, send_counts: List[int], device) -> List[int]:
        s = torch.tensor(send_counts, dtype=torch.int64, device="cpu" if self.host else device)
        r = torch.empty_like(s)
        self.dist.all_to_all_single(r, s, group=self.group)
        return [int(v) for v in r.cpu().tolist()]

    def counts_from_device(self, totals: torch.Tensor):
        """(send counts, receive counts) from this rank's device totals, with
        a single host read: the counts are exchanged before they are read."""
        s = totals.cpu() if self.host else totals
        r = torch.empty_like(s)
        self.dist.all_to_all_single(r, s, group=self.group)
        both = torch.cat([s, r]).cpu().tolist()
        n = len(both) // 2
        return [int(v) for v in both[:n]], [int(v) for v in both[n:]]

    def row_costs(self, local: np.ndarray) -> np.ndarray:
        """The sum over ranks of their band row costs (each rank fills its rows)."""
        t = torch.from_numpy(np.ascontiguousarray(local, np.float64))
        if not self.host:
            t = t.cuda()
        self.dist.all_reduce(t, group=self.group)
        return t.cpu().numpy()

    def payload(self, send: torch.Tensor, send_rows: List[int], recv_rows: List[int], row_elems: int):
        src = send.reshape(-1)
        dev = src.device
        if self.host:
            src = src.cpu()
        out = torch.empty((sum(recv_rows) * row_elems,), dtype=src.dtype, device=src.device)
        self.dist.all_to_all_single(out, src, output_split_sizes=[r * row_elems for r in recv_rows],
                                    input_split_sizes=[r * row_elems for r in send_rows], group=self.group)
        return out.to(dev) if self.host else out


def render_distributed(rank_state: InterleavedRank, ex: DistExchange, params: GaussianParams, cam, bg,
                       dL_dimage: Optional[torch.Tensor] = None):
    """One view on this rank of a group: forward (and backward when dL_dimage
    is given). Returns (band image, local parameter gradients or None)."""
    rank_state.project(params, cam)
    counts, recv_counts = ex.counts_from_device(rank_state.totals)  # the view's one host round trip
    send = rank_state.pack(counts)
    recv = ex.payload(send, counts, recv_counts, WIRE)
    img = rank_state.receive_and_render(recv, recv_counts, cam, bg)
    if dL_dimage is None:
        return img, None
    back, back_counts = rank_state.backward_band(dL_dimage)
    ret = ex.payload(back.reshape(-1), back_counts, counts, 12)
    return img, rank_state.finish_backward(ret.reshape(-1, 12))


def emulate(ranks: List[InterleavedRank], params: List[GaussianParams], cam, bg,
            dL_dimage: Optional[torch.Tensor] = None):
    """All ranks of a group in this process on one GPU: the exchanges are
    device copies. Returns (the composed image [3][H][W], per-rank local
    parameter gradients or None)."""
    G = len(ranks)
    packs = [r.project_and_pack(p, cam) for r, p in zip(ranks, params)]
    offs = []
    for send, counts in packs:
        o = [0]
        for v in counts:
            o.append(o[-1] + v)
        offs.append(o)
    image = None
    for q, rq in enumerate(ranks):
        parts = [packs[s][0][offs[s][q] * WIRE: offs[s][q + 1] * WIRE] for s in range(G)]
        recv = torch.cat(parts) if parts else torch.empty(0, dtype=torch.uint8, device=rq.dev)
        img = rq.receive_and_render(recv, [packs[s][1][q] for s in range(G)], cam, bg)
        if image is None:
            image = torch.empty_like(img)
        lo, hi = rq.row_lo * 16, min(rq.row_hi * 16, rq.H)
        image[:, lo:hi] = img[:, lo:hi]
    if dL_dimage is None:
        return image, None
    backs = [rq.backward_band(dL_dimage) for rq in ranks]
    grads = []
    for s, rs in enumerate(ranks):
        rows = []
        for q in range(G):
            back, recv_counts = backs[q]
            start = sum(recv_counts[:s])
            rows.append(back[start: start + recv_counts[s]])
        ret = torch.cat(rows) if rows else torch.empty((0, 12), device=rs.dev)
        grads.append(rs.finish_backward(ret.contiguous()))
    return image, grads
