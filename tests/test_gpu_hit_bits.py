"""The forward's hit bytes (one per sorted list entry: the 8x4 pixel blocks
of its tile where it blended) and the backward that walks only them.

- Every entry up to a tile's deepest last blend gets a byte (the same bytes
  whatever the buffer held before).
- The block of every pixel has its bit set at the pixel's last blend, and
  each pixel's block has at least n_contrib set bits before its last.
- The backward gives the oracle's gradients within the suite's tolerance
  with the bytes and without them (its own region tests), and the forward
  outputs do not depend on whether the bytes are written."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, Rasterizer
from tests.gpu_helpers import assert_bits, grad_tol_check

pytestmark = pytest.mark.gpu

NAMES = ["means", "log_scales", "quats", "opacity_logits", "sh"]


def _forward(sc, pose=0, use_hits=True, fill=None):
    cam = sc.cameras[pose]
    R = Rasterizer(sc.N, sc.sh_degree, cam.width, cam.height)
    R.use_hit_bits = use_hits
    if fill is not None:
        R.hit_bits.fill_(fill)
    R.forward(GaussianParams.from_scene(sc), cam, sc.bg)
    torch.cuda.synchronize()
    return R


def _tile_of_pixels(W, H):
    TW = (W + 15) // 16
    v, u = np.mgrid[0:H, 0:W]
    return (v // 16) * TW + (u // 16), ((v % 16) // 4) * 2 + (u % 16) // 8


@pytest.mark.parametrize("seed,W,H", [(150, 173, 95), (151, 64, 64), (152, 300, 41)])
def test_hit_bytes_written_and_set_at_each_last_blend(seed, W, H):
    sc = S.random_scene(3000, W, H, sh_degree=1, seed=seed, log_scale=(-2.6, 0.4))
    Ra = _forward(sc, fill=0x00)
    Rb = _forward(sc, fill=0xFF)
    ranges = Ra.ranges.cpu().numpy().view(np.uint32).astype(np.int64)
    last = Ra.last.cpu().numpy()
    ha, hb = Ra.hit_bits.cpu().numpy(), Rb.hit_bits.cpu().numpy()
    tile, block = _tile_of_pixels(W, H)
    # deepest last blend per tile: every entry before it has a byte
    deep = np.zeros(ranges.shape[0], np.int64)
    np.maximum.at(deep, tile.ravel(), last.ravel())
    for t in np.nonzero(deep)[0]:
        s0 = ranges[t, 0]
        assert np.array_equal(ha[s0: s0 + deep[t]], hb[s0: s0 + deep[t]]), f"tile {t}: bytes not written"
    # the block of each pixel may blend the entry it blended last
    ys, xs = np.nonzero(last > 0)
    entry = ranges[tile[ys, xs], 0] + last[ys, xs] - 1
    bits = (ha[entry] >> block[ys, xs]) & 1
    assert bits.all(), f"{int((bits == 0).sum())} last blends outside their block's bits"
    assert len(ys) > 1000
    # every blend of a pixel is an entry with its block's bit: per pixel, the
    # set bits of its block among entries [0, last) are at least n_contrib
    nc = Ra.n_contrib.cpu().numpy()
    for y, x in list(zip(ys, xs))[::97]:
        s0 = ranges[tile[y, x], 0]
        setb = int(((ha[s0: s0 + last[y, x]] >> block[y, x]) & 1).sum())
        assert setb >= nc[y, x], (y, x, setb, nc[y, x])


@pytest.mark.parametrize("name", ["ragged", "dense_sh3"])
def test_backward_with_and_without_hit_bytes(name):
    if name == "ragged":
        sc = S.random_scene(2500, 173, 95, sh_degree=2, seed=153, log_scale=(-2.5, 0.4))
    else:
        sc = S.random_scene(6000, 128, 112, sh_degree=3, seed=154, log_scale=(-2.0, 0.6))
    cam = sc.cameras[0]
    ref = oracle.render(sc)
    ob = oracle.backward(sc, cam, ref["rec"], ref["bins"], sc.grad_image(0))
    g = torch.from_numpy(sc.grad_image(0)).cuda()
    outs = {}
    for use in (True, False):
        R = _forward(sc, use_hits=use)
        assert_bits(R.image.cpu().numpy(), ref["fwd"]["image"], f"image hits={use}")
        assert_bits(R.last.cpu().numpy(), ref["fwd"]["last"], f"last hits={use}")
        grads = R.backward(g)
        torch.cuda.synchronize()
        outs[use] = {n: grads[n].cpu().numpy().copy() for n in NAMES}
        for n in NAMES:
            grad_tol_check(outs[use][n], ob["d_" + n], ob["m_" + n], what=f"{n} hits={use}")


def test_stale_hit_bytes_are_not_used():
    # a backward after a new bin sort without a forward falls back to the
    # kernel's own region tests (the bytes belong to the previous lists)
    sc = S.random_scene(1500, 96, 80, sh_degree=1, seed=155, n_poses=2)
    R = _forward(sc, pose=0)
    assert R._hits_in() is not None
    R.bin_sort(R.cam)
    assert R._hits_in() is None
