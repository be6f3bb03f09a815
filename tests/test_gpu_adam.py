"""Quantised SH Adam on the GPU (gs_quant_encode/decode, gs_adam_sh_quant)
against the oracle: codes bit-exact (integers decided in the same fp32
arithmetic on both sides), bounds bit-exact (min and max of identical fp32
values), decoded values bit-exact."""

import numpy as np
import pytest
import torch

import oracle
from differentiable_tile_rasterizer_b200 import gs, synthetic as S
from differentiable_tile_rasterizer_b200.pipeline import GaussianParams, QuantizedSHAdam, Rasterizer
from tests.gpu_helpers import assert_bits

pytestmark = pytest.mark.gpu

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-15, scale=1e-15)


def _planes(rng, U, N):
    x = rng.normal(0, 0.2, (U, N)).astype(np.float32)
    x[0, :300] = 0.25  # a constant block and a part of the next
    return x


def _grads(rng, U, N):
    return (rng.normal(0, 1e-3, (U, N)) * 10.0 ** rng.uniform(-3, 1, (U, N))).astype(np.float32)


@pytest.mark.parametrize("bits,N", [(16, 1000), (8, 1000), (16, 256), (8, 37)])
def test_encode_decode_bitexact(bits, N):
    rng = np.random.default_rng(100 + bits + N)
    U = 7
    x = _planes(rng, U, N)
    codes_ref, bounds_ref = oracle.quant_encode(x, bits)
    nblk = (N + 255) // 256
    ct = torch.int16 if bits == 16 else torch.uint8
    codes = torch.full((U, nblk * 256), 77, dtype=ct, device="cuda")
    bounds = torch.zeros((U, nblk, 2), dtype=torch.float32, device="cuda")
    gs.gs_quant_encode(torch.from_numpy(x).cuda(), U, N, bits, codes, bounds)
    xd = torch.zeros((U, N), dtype=torch.float32, device="cuda")
    gs.gs_quant_decode(codes, bounds, U, N, bits, xd)
    torch.cuda.synchronize()
    got = codes.cpu().numpy().view(np.uint16 if bits == 16 else np.uint8).astype(np.uint32)
    assert_bits(got, codes_ref, "codes")
    assert_bits(bounds.cpu().numpy(), bounds_ref, "bounds")
    assert_bits(xd.cpu().numpy(), oracle.quant_decode(codes_ref, bounds_ref, N, bits), "decoded")


def _gpu_state(st):
    return {"pc": torch.from_numpy(st["pc"].astype(np.uint16).view(np.int16)).cuda(),
            "mc": torch.from_numpy(st["mc"].astype(np.uint8)).cuda(),
            "vc": torch.from_numpy(st["vc"].astype(np.uint8)).cuda(),
            "pb": torch.from_numpy(st["pb"].copy()).cuda(), "mb": torch.from_numpy(st["mb"].copy()).cuda(),
            "vb": torch.from_numpy(st["vb"].copy()).cuda()}


def _compare(g, st, what):
    assert_bits(g["pc"].cpu().numpy().view(np.uint16).astype(np.uint32), st["pc"], what + " value codes")
    assert_bits(g["mc"].cpu().numpy().astype(np.uint32), st["mc"], what + " m codes")
    assert_bits(g["vc"].cpu().numpy().astype(np.uint32), st["vc"], what + " v codes")
    for k in ("pb", "mb", "vb"):
        assert_bits(g[k].cpu().numpy(), st[k], what + " " + k)


@pytest.mark.parametrize("U,N", [(9, 1000), (45, 4096 + 77)])
def test_adam_steps_bitexact(U, N):
    rng = np.random.default_rng(110 + N)
    x = _planes(rng, U, N)
    pc, pb = oracle.quant_encode(x, 16)
    z = np.zeros((U, N), np.float32)
    mc, mb = oracle.quant_encode(z, 8)
    vc, vb = oracle.quant_encode(z, 8)
    st = {"pc": pc, "pb": pb, "mc": mc, "mb": mb, "vc": vc, "vb": vb}
    g = _gpu_state(st)
    for step in range(1, 5):
        gr = _grads(rng, U, N)
        oracle.adam_sh_quant(gr, st, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["scale"], step)
        gs.gs_adam_sh_quant(torch.from_numpy(gr).cuda(), U, N, g["pc"], g["pb"], g["mc"], g["mb"], g["vc"], g["vb"],
                            HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["scale"], step)
        torch.cuda.synchronize()
        _compare(g, st, f"step {step}")


def test_adam_after_a_real_backward():
    # gradients of a rendered view (SH3): the optimizer holds planes 3..47
    sc = S.random_scene(3000, 96, 72, sh_degree=3, seed=111)
    cam = sc.cameras[0]
    R = Rasterizer(sc.N, 3, cam.width, cam.height, capacity=64 * sc.N)
    params = GaussianParams.from_scene(sc)
    R.forward(params, cam, sc.bg)
    R.backward(torch.from_numpy(sc.grad_image(0)).cuda())
    opt = QuantizedSHAdam(sc.N, 3, lr=1e-3, eps=1e-15, code_scale=1e-15)
    opt.load(params.sh)
    x = params.sh.cpu().numpy()[3:]
    pc, pb = oracle.quant_encode(x, 16)
    z = np.zeros_like(x)
    mc, mb = oracle.quant_encode(z, 8)
    vc, vb = oracle.quant_encode(z, 8)
    st = {"pc": pc, "pb": pb, "mc": mc, "mb": mb, "vc": vc, "vb": vb}
    d_sh = R.grads["sh"]
    opt.step(d_sh)
    torch.cuda.synchronize()
    oracle.adam_sh_quant(d_sh.cpu().numpy()[3:], st, 1e-3, 0.9, 0.999, 1e-15, 1e-15, 1)
    _compare({"pc": opt.pc, "pb": opt.pb, "mc": opt.mc, "mb": opt.mb, "vc": opt.vc, "vb": opt.vb}, st, "step 1")
    # decoded values back into the SH planes for the next render
    sh = params.sh.clone()
    opt.store(sh)
    torch.cuda.synchronize()
    assert_bits(sh.cpu().numpy()[3:], oracle.quant_decode(st["pc"], st["pb"], sc.N, 16), "stored SH")
    assert_bits(sh.cpu().numpy()[:3], params.sh.cpu().numpy()[:3], "DC planes untouched")


def test_adam_argument_checks():
    t = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(gs.GsError):
        gs.gs_quant_encode(t, 1, 16, 12, t, t)  # bits
    with pytest.raises(gs.GsError):
        gs.gs_adam_sh_quant(t, 1, 16, t, t, t, t, t, t, 1e-3, 0.9, 0.999, 1e-15, 1e-15, 0)  # step 0


@pytest.mark.parametrize("U,N,off", [(5, 3 * 256 + 100, 1), (3, 512, 3), (4, 1001, 2)])
def test_adam_unaligned_buffers_take_the_scalar_path(U, N, off):
    # codes and gradients at odd element offsets into larger buffers: not
    # 16/8-byte aligned, so the kernel takes its element-wise loads and stores
    rng = np.random.default_rng(120 + off)
    x = _planes(rng, U, N)
    pc, pb = oracle.quant_encode(x, 16)
    z = np.zeros((U, N), np.float32)
    mc, mb = oracle.quant_encode(z, 8)
    vc, vb = oracle.quant_encode(z, 8)
    st = {"pc": pc, "pb": pb, "mc": mc, "mb": mb, "vc": vc, "vb": vb}
    g = _gpu_state(st)
    L = pc.size

    def shifted(t):
        big = torch.zeros(L + 16, dtype=t.dtype, device="cuda")
        v = big[off: off + L]
        v.copy_(t.reshape(-1))
        return v

    sp, sm, sv = shifted(g["pc"]), shifted(g["mc"]), shifted(g["vc"])
    assert sp.data_ptr() % 16 and sm.data_ptr() % 8
    for step in range(1, 4):
        gr = _grads(rng, U, N)
        gbig = torch.zeros(U * N + 8, dtype=torch.float32, device="cuda")
        gt = gbig[off: off + U * N]
        gt.copy_(torch.from_numpy(gr.reshape(-1)))
        oracle.adam_sh_quant(gr, st, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["scale"], step)
        gs.gs_adam_sh_quant(gt, U, N, sp, g["pb"], sm, g["mb"], sv, g["vb"],
                            HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["scale"], step)
        torch.cuda.synchronize()
        _compare({"pc": sp.view(U, -1), "mc": sm.view(U, -1), "vc": sv.view(U, -1), "pb": g["pb"], "mb": g["mb"],
                  "vb": g["vb"]}, st, f"step {step}")
