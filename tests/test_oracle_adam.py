"""Pins for the oracle's quantised SH Adam step (Spirula Studio page: 16-bit
block codes of the SH values, 8-bit block codes of log1p-transformed Adam
moments, one (min, max) pair per 256 units).

References that are not the oracle: float64 numpy logarithms and
exponentials of the same (rounded) arguments, the error bound of a linear
code (half a step), and a float64 textbook Adam step run from the decoded
state, compared through the new codes' step sizes."""

import numpy as np
import pytest

import oracle

F32 = np.float32
L2E = float(F32(1.0 / np.log(2.0)))


def _ulp_err(got, ref):
    return abs(float(got) - ref) / np.spacing(F32(abs(ref) if ref else 1e-30))


def test_log2_spec_against_float64():
    rng = np.random.default_rng(90)
    ys = np.concatenate([np.float32(2.0) ** rng.uniform(0, 100, 4000), [1.0, 2.0, 1.4142135, 1.4142137, 3e38]])
    # measured 2.2 ulp at most (the last rounding of e + s p when m < 1
    # cancels); the result feeds an 8-bit code, far coarser
    worst = max(_ulp_err(oracle.log2_spec(y), np.log2(np.float64(F32(y)))) for y in ys)
    assert worst <= 3.0, worst
    assert oracle.log2_spec(1.0) == 0.0 and oracle.log2_spec(1024.0) == 10.0
    assert oracle.log2_spec(float("inf")) == float("inf")


def test_log1p_and_expm1_spec_against_float64():
    rng = np.random.default_rng(91)
    for z in np.concatenate([10.0 ** rng.uniform(-6, 20, 3000), [0.0, 1.0]]).astype(np.float32):
        u = np.float64(F32(1.0) + z)  # the definition logs the rounded 1 + z
        ref = np.log(u)
        assert _ulp_err(oracle.log1p_spec(z), ref) <= 3.0, z
    for y in rng.uniform(0, 60, 3000).astype(np.float32):
        ref = np.exp2(np.float64(F32(y * F32(L2E)))) - 1.0
        got = oracle.expm1_spec(y)
        # exp2 within 1 ulp of its argument's exact value, then one rounding
        assert abs(got - ref) <= 2.0 * float(np.spacing(F32(ref + 1.0))), y
    assert oracle.expm1_spec(0.0) == 0.0


def _check_block_codes(x, bits):
    U, N = x.shape
    nb = (N + 255) // 256
    codes, bounds = oracle.quant_encode(x, bits)
    Q = 2 ** bits - 1
    assert codes.shape == (U, 256 * nb) and bounds.shape == (U, nb, 2)
    xh = oracle.quant_decode(codes, bounds, N, bits)
    for u in range(U):
        for b in range(nb):
            sl = slice(256 * b, min(N, 256 * b + 256))
            blk, c = x[u, sl], codes[u, sl]
            lo, hi = bounds[u, b]
            assert lo == blk.min() and hi == blk.max()
            d = float(hi) - float(lo)
            if d == 0:
                assert not c.any() and np.all(xh[u, sl] == lo)
                continue
            assert c[np.argmin(blk)] == 0 and c[np.argmax(blk)] == Q
            o = np.argsort(blk, kind="stable")
            assert np.all(np.diff(c[o].astype(np.int64)) >= 0)  # order kept
            err = np.abs(xh[u, sl].astype(np.float64) - blk)
            assert err.max() <= d / (2 * Q) * (1 + 1e-3) + 4 * np.spacing(F32(max(abs(lo), abs(hi))))
    assert not codes[:, N:].any()  # padding


@pytest.mark.parametrize("bits", [8, 16])
def test_block_code_error_bound_and_order(bits):
    rng = np.random.default_rng(92 + bits)
    U, N = 5, 1000  # 4 blocks, the last one ragged
    x = rng.normal(0, 1, (U, N)).astype(np.float32) * (10.0 ** rng.uniform(-4, 2, (U, 1))).astype(np.float32)
    x[2, 256:512] = 0.375  # a constant block
    _check_block_codes(x, bits)


def test_block_codes_on_random_planes():
    # plane counts, ragged widths, scales, offsets and constant runs drawn by
    # hypothesis: the same bounds, extremes, order and half-step error
    from hypothesis import given, settings
    from hypothesis import strategies as st

    @settings(max_examples=40, deadline=None)
    @given(st.integers(1, 4), st.integers(1, 700), st.sampled_from([8, 16]), st.floats(-6, 3),
           st.floats(-100, 100), st.integers(0, 2 ** 16), st.booleans())
    def check(U, N, bits, log_scale, offset, seed, constant_run):
        rng = np.random.default_rng(seed)
        x = (rng.normal(0, 1, (U, N)) * 10.0 ** log_scale + offset).astype(np.float32)
        if constant_run:
            x[0, : min(N, 300)] = np.float32(offset)
        _check_block_codes(x, bits)

    check()


def _decode_state(st, N):
    p = oracle.quant_decode(st["pc"], st["pb"], N, 16).astype(np.float64)
    ym = oracle.quant_decode(st["mc"], st["mb"], N, 8).astype(np.float64)
    yv = oracle.quant_decode(st["vc"], st["vb"], N, 8).astype(np.float64)
    return p, ym, yv


def test_adam_step_against_float64_textbook():
    rng = np.random.default_rng(93)
    U, N = 6, 700
    lr, b1, b2, eps, e = 1e-3, 0.9, 0.999, 1e-15, 1e-15
    x0 = rng.normal(0, 0.3, (U, N)).astype(np.float32)
    pc, pb = oracle.quant_encode(x0, 16)
    zeros = np.zeros((U, N), np.float32)
    mc, mb = oracle.quant_encode(zeros, 8)
    vc, vb = oracle.quant_encode(zeros, 8)
    st = {"pc": pc, "pb": pb, "mc": mc, "mb": mb, "vc": vc, "vb": vb}
    for step in (1, 2, 3):
        g = (rng.normal(0, 1e-3, (U, N)) * 10.0 ** rng.uniform(-2, 1, (U, N))).astype(np.float64)
        p, ym, yv = _decode_state(st, N)
        m = np.sign(ym) * e * np.expm1(np.abs(ym))
        v = (e * np.expm1(yv)) ** 2
        g32 = g.astype(np.float32).astype(np.float64)
        m1 = b1 * m + (1 - b1) * g32
        v1 = b2 * v + (1 - b2) * g32 ** 2
        p1 = p - lr * (m1 / (1 - b1 ** step)) / (np.sqrt(v1 / (1 - b2 ** step)) + eps)
        oracle.adam_sh_quant(g32.astype(np.float32), st, lr, b1, b2, eps, e, step)
        pn, ymn, yvn = _decode_state(st, N)
        nb = (N + 255) // 256
        for u in range(U):
            for b in range(nb):
                sl = slice(256 * b, min(N, 256 * b + 256))
                dp = float(st["pb"][u, b, 1] - st["pb"][u, b, 0])
                assert np.abs(pn[u, sl] - p1[u, sl]).max() <= dp / (2 * 65535) + 2e-6 * np.abs(p1[u, sl]).max()
                ref_ym = np.sign(m1[u, sl]) * np.log1p(np.abs(m1[u, sl]) / e)
                ref_yv = np.log1p(np.sqrt(v1[u, sl]) / e)
                dm = float(st["mb"][u, b, 1] - st["mb"][u, b, 0])
                dv = float(st["vb"][u, b, 1] - st["vb"][u, b, 0])
                # half a code step, plus the fp32 log of a value known to ~1e-6
                assert np.abs(ymn[u, sl] - ref_ym).max() <= dm / (2 * 255) + 1e-4, (step, u, b)
                assert np.abs(yvn[u, sl] - ref_yv).max() <= dv / (2 * 255) + 1e-4, (step, u, b)
    assert np.abs(pn - x0).max() > 1e-3  # the values did move
