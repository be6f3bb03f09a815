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

from typing import List, Optional

import torch

from . import gs
from .pipeline import GaussianParams, Rasterizer

WIRE = gs.GS_WIRE_RECORD_BYTES


def band_rows(rank: int, world: int, tiles_y: int):
    """Tile rows [lo, hi) owned by `rank`."""
    return rank * tiles_y // world, (rank + 1) * tiles_y // world


def local_params(params: GaussianParams, rank: int, world: int) -> GaussianParams:
    """The Gaussians rank `rank` holds: global indices rank, rank + world, ..."""
    pick = lambda t: t[..., rank::world].contiguous()
    imp = None if params.importance is None else pick(params.importance)
    return GaussianParams(pick(params.means), pick(params.log_scales), pick(params.quats),
                          pick(params.opacity_logits), pick(params.sh), params.sh_degree, imp)


class InterleavedRank:
    def __init__(self, n_local: int, sh_degree: int, width: int, height: int, rank: int, world: int,
                 device=None, recv_capacity: Optional[int] = None):
        if not 1 <= world <= gs.GS_MAX_RANKS or not 0 <= rank < world:
            raise ValueError("bad rank / world")
        self.rank, self.world = rank, world
        self.dev = torch.device(device or "cuda")
        self.local = Rasterizer(n_local, sh_degree, width, height, device=self.dev)
        self.row_lo, self.row_hi = band_rows(rank, world, self.local.TH)
        self.sh_degree, self.W, self.H = sh_degree, width, height
        self._band_cap = 0
        self.band: Optional[Rasterizer] = None
        self._ensure_band(recv_capacity or max(2 * n_local, 1024))
        nc = int(gs.load().gs_route_ctas(max(n_local, 1)))
        self.mask = torch.empty(max(n_local, 1), dtype=torch.int32, device=self.dev)
        self.cta_counts = torch.empty(nc * world, dtype=torch.int32, device=self.dev)
        self.totals = torch.empty(world, dtype=torch.int64, device=self.dev)

    def _ensure_band(self, n: int):
        if n <= self._band_cap:
            return
        cap = int(n * 1.25) + 1024
        self.band = Rasterizer(cap, self.sh_degree, self.W, self.H, device=self.dev, capacity=8 * cap)
        self._band_cap = cap

    # ---------------------------------------------------------------- forward
    def project_and_pack(self, params: GaussianParams, cam, lod_dist=0.0):
        """Preprocess the local Gaussians and pack the wire records for every
        rank. Returns (send bytes [sum counts * 64] uint8, counts per rank)."""
        c = cam if isinstance(cam, gs.GsCamera) else gs.camera(cam)
        L = self.local
        L.params, L.cam = params, c
        L.culled = False
        L.preprocess(params, c)
        n = L.N
        gs.gs_route_count(L._proj, n, self.world, L.TH, self.mask, self.cta_counts, self.totals)
        counts = [int(v) for v in self.totals.cpu().tolist()]
        offs = [0]
        for v in counts:
            offs.append(offs[-1] + v)
        self.sent = offs[-1]
        dst = torch.tensor(offs[:-1], dtype=torch.int64, device=self.dev)
        send = torch.empty(max(self.sent, 1) * WIRE, dtype=torch.uint8, device=self.dev)
        self.src_idx = torch.empty(max(self.sent, 1), dtype=torch.int32, device=self.dev)
        gs.gs_route_pack(L._proj, self.mask, n, self.world, self.rank, self.cta_counts, dst, send, self.src_idx)
        self.send_counts = counts
        return send[: self.sent * WIRE], counts

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
    payload (wire records forward, gradient rows backward)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group

    def counts(self, send_counts: List[int], device) -> List[int]:
        s = torch.tensor(send_counts, dtype=torch.int64, device=device)
        r = torch.empty_like(s)
        self.dist.all_to_all_single(r, s, group=self.group)
        return [int(v) for v in r.cpu().tolist()]

    def payload(self, send: torch.Tensor, send_rows: List[int], recv_rows: List[int], row_elems: int):
        out = torch.empty((sum(recv_rows) * row_elems,), dtype=send.dtype, device=send.device)
        self.dist.all_to_all_single(out, send.reshape(-1), output_split_sizes=[r * row_elems for r in recv_rows],
                                    input_split_sizes=[r * row_elems for r in send_rows], group=self.group)
        return out


def render_distributed(rank_state: InterleavedRank, ex: DistExchange, params: GaussianParams, cam, bg,
                       dL_dimage: Optional[torch.Tensor] = None):
    """One view on this rank of a group: forward (and backward when dL_dimage
    is given). Returns (band image, local parameter gradients or None)."""
    send, counts = rank_state.project_and_pack(params, cam)
    recv_counts = ex.counts(counts, send.device)
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
