"""Pins for the spherical-harmonic colour basis.

The basis is the real orthonormal one built from the complex harmonics with
the Condon-Shortley phase (scipy.special.sph_harm_y):
  m < 0: sqrt(2) Im Y_l^|m|,  m = 0: Y_l^0,  m > 0: sqrt(2) Re Y_l^m,
ordered l = 0..3, m = -l..l.
"""

import numpy as np
from scipy.special import sph_harm_y


def _scipy_real_sh(d):
    theta = np.arccos(np.clip(d[:, 2], -1, 1))
    phi = np.arctan2(d[:, 1], d[:, 0])
    cols = []
    for l in range(4):
        for m in range(-l, l + 1):
            if m < 0:
                cols.append(np.sqrt(2) * np.imag(sph_harm_y(l, -m, theta, phi)))
            elif m == 0:
                cols.append(np.real(sph_harm_y(l, 0, theta, phi)))
            else:
                cols.append(np.sqrt(2) * np.real(sph_harm_y(l, m, theta, phi)))
    return np.stack(cols, 1)


def _dirs(n, seed):
    d = np.random.default_rng(seed).standard_normal((n, 3))
    return d / np.linalg.norm(d, axis=1, keepdims=True)


def test_basis_matches_scipy(orc):
    d = _dirs(4000, 0)
    assert np.abs(orc.sh_basis(d) - _scipy_real_sh(d)).max() < 1e-13


def test_basis_fp32_close_to_fp64(orc):
    d = _dirs(4000, 1).astype(np.float32)
    y32 = orc.sh_basis(d, np.float32)
    y64 = orc.sh_basis(d.astype(np.float64))
    assert np.abs(y32 - y64).max() < 5e-6


def test_orthonormal_by_quadrature(orc):
    # Gauss-Legendre in cos(theta) x uniform in phi: exact for the degree-6
    # products Y_i Y_j.
    x, w = np.polynomial.legendre.leggauss(8)
    nphi = 16
    phi = 2 * np.pi * np.arange(nphi) / nphi
    ct, ph = np.meshgrid(x, phi, indexing="ij")
    st = np.sqrt(1 - ct ** 2)
    d = np.stack([st * np.cos(ph), st * np.sin(ph), ct], -1).reshape(-1, 3)
    wt = (w[:, None] * np.full(nphi, 2 * np.pi / nphi)[None, :]).reshape(-1)
    Y = orc.sh_basis(d)
    gram = (Y * wt[:, None]).T @ Y
    assert np.abs(gram - np.eye(16)).max() < 1e-13


def test_basis_gradient_by_central_differences(orc):
    d = _dirs(200, 3)
    G = orc.sh_basis_grad(d)
    h = 1e-6
    for m in range(3):
        e = np.zeros(3)
        e[m] = h
        # the basis is a polynomial in (x, y, z); differentiate it off the sphere
        num = (orc.sh_basis(d + e) - orc.sh_basis(d - e)) / (2 * h)
        assert np.abs(num - G[:, :, m]).max() < 1e-8
