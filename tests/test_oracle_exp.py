"""Pins for the oracle's constants and its software exp2.

The constants are checked against exact values computed here with Python's
decimal module; exp2 against libm's double-precision exp2 rounded to fp32.
"""

import decimal
import math

import numpy as np
import pytest

D = decimal.Decimal
decimal.getcontext().prec = 60


def _f32(x: D) -> np.float32:
    v = float(x)  # correctly rounded to double
    return np.float32(v)


def _ln2() -> D:
    return D(2).ln()


def test_taylor_coefficients_exact(orc):
    c = orc.constants()["exp2_taylor"]
    ln2 = _ln2()
    for k in range(8):
        exact = ln2 ** k / D(math.factorial(k))
        assert c[k] == _f32(exact), k


def test_log2e_and_conic_scale(orc):
    c = orc.constants()
    l2e = D(1) / _ln2()
    assert c["log2e"] == _f32(l2e)
    assert c["kh"] == _f32(-l2e / 2)
    assert c["kf"] == _f32(-l2e)
    assert c["kf"] == 2 * c["kh"]


def test_thresholds(orc):
    c = orc.constants()
    assert c["alpha_min"] == _f32(D(1) / D(255))
    assert c["alpha_max"] == np.float32(0.99)
    assert c["t_min"] == np.float32(1e-4)
    assert c["dilation"] == np.float32(0.3)


def test_sh_constants_closed_form(orc):
    sh = orc.constants()["sh"]
    pi = D("3.14159265358979323846264338327950288419716939937510")
    r = lambda x: x.sqrt()
    want = [
        D(1) / (2 * r(pi)),
        -r(D(3) / (4 * pi)), r(D(3) / (4 * pi)), -r(D(3) / (4 * pi)),
        r(D(15) / pi) / 2, -r(D(15) / pi) / 2, r(D(5) / pi) / 4, -r(D(15) / pi) / 2,
        r(D(15) / pi) / 4,
        -r(D(35) / (2 * pi)) / 4, r(D(105) / pi) / 2, -r(D(21) / (2 * pi)) / 4,
        r(D(7) / pi) / 4, -r(D(21) / (2 * pi)) / 4, r(D(105) / pi) / 4,
        -r(D(35) / (2 * pi)) / 4,
    ]
    for k in range(16):
        assert sh[k] == _f32(want[k]), k


def _ulp_err(got: np.ndarray, ref64: np.ndarray) -> np.ndarray:
    ref32 = ref64.astype(np.float32)
    ulp = np.spacing(np.abs(ref32)).astype(np.float64)
    return np.abs(got.astype(np.float64) - ref64) / ulp


def test_exp2_accuracy_dense(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.uniform(-125.0, 127.0, 2_000_000),
        rng.uniform(-30.0, 2.0, 2_000_000),   # the range alpha uses
        rng.uniform(-1.0, 1.0, 1_000_000),
    ]).astype(np.float32)
    y = orc.exp2(x)
    err = _ulp_err(y, np.exp2(x.astype(np.float64)))
    # Taylor truncation < 0.05 ulp; Horner in fp32 adds < 1.5 ulp.
    assert err.max() <= 2.0, err.max()
    assert np.mean(err <= 0.5) > 0.9


def test_exp2_special_cases(orc):
    ints = np.arange(-125, 128, dtype=np.float32)
    assert np.array_equal(orc.exp2(ints), np.ldexp(np.float32(1), ints.astype(np.int32)))
    y = orc.exp2(np.array([-125.5, -200.0, np.nan, -np.inf, 127.5, np.inf, 0.0, -0.0], np.float32))
    assert y[0] == 0 and y[1] == 0 and y[2] == 0 and y[3] == 0
    assert np.isinf(y[4]) and np.isinf(y[5])
    assert y[6] == 1.0 and y[7] == 1.0


def test_exp2_monotone_on_alpha_range(orc):
    x = np.sort(np.random.default_rng(2).uniform(-12.0, 0.5, 500_000).astype(np.float32))
    y = orc.exp2(x)
    assert np.all(np.diff(y) >= 0)
