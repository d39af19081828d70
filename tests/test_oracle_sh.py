"""Pins of the oracle's real spherical harmonics (oracle/sh.py) against facts outside it.

Reading fixed by the oracle: component normalisation, no Condon-Shortley phase,
m = -l..l with Y_{l,m>0} ~ cos(m phi) and Y_{l,m<0} ~ sin(|m| phi).
"""
import numpy as np
import pytest
import scipy.special as sps

from oracle import sh


def _dirs(n, seed=0):
    rng = np.random.default_rng(seed)
    r = rng.standard_normal((n, 3))
    return r * rng.uniform(0.3, 3.0, size=(n, 1))


def test_closed_forms_l0_l1_l2():
    r = _dirs(50)
    u = r / np.linalg.norm(r, axis=1, keepdims=True)
    x, y, z = u.T
    Y = sh.sh(2, r)
    assert np.allclose(Y[:, 0], 1.0, atol=1e-15)
    s3 = np.sqrt(3.0)
    assert np.allclose(Y[:, 1:4], s3 * np.stack([y, z, x], 1), atol=1e-14)
    s15, s5 = np.sqrt(15.0), np.sqrt(5.0)
    want = np.stack([s15 * x * y, s15 * y * z, s5 / 2 * (3 * z * z - 1), s15 * x * z,
                     s15 / 2 * (x * x - y * y)], 1)
    assert np.allclose(Y[:, 4:9], want, atol=1e-13)


@pytest.mark.parametrize("l", range(0, 6))
def test_against_scipy_complex_harmonics(l):
    """Real form from scipy's orthonormal complex Y_l^m (which carries the (-1)^m phase)."""
    r = _dirs(40, seed=l)
    u = r / np.linalg.norm(r, axis=1, keepdims=True)
    theta = np.arccos(np.clip(u[:, 2], -1, 1))
    phi = np.mod(np.arctan2(u[:, 1], u[:, 0]), 2 * np.pi)
    ours = sh.sh_block(l, r)
    scale = np.sqrt(4 * np.pi)
    for i, m in enumerate(range(-l, l + 1)):
        mu = abs(m)
        yc = sps.sph_harm_y(l, mu, theta, phi)
        if m == 0:
            ref = scale * yc.real
        elif m > 0:
            ref = scale * np.sqrt(2) * (-1) ** mu * yc.real
        else:
            ref = scale * np.sqrt(2) * (-1) ** mu * yc.imag
        assert np.allclose(ours[:, i], ref, atol=1e-11), (l, m)


@pytest.mark.parametrize("l", range(0, 6))
def test_norm_and_addition_theorem(l):
    a, b = _dirs(30, 1), _dirs(30, 2)
    Ya, Yb = sh.sh_block(l, a), sh.sh_block(l, b)
    assert np.allclose(np.sum(Ya**2, axis=1), 2 * l + 1, atol=1e-11)
    cosg = np.sum(a * b, 1) / np.linalg.norm(a, axis=1) / np.linalg.norm(b, axis=1)
    assert np.allclose(np.sum(Ya * Yb, axis=1), (2 * l + 1) * sps.eval_legendre(l, cosg), atol=1e-11)


@pytest.mark.parametrize("l", range(0, 5))
def test_parity_and_scale_invariance(l):
    r = _dirs(20, 3)
    assert np.allclose(sh.sh_block(l, -r), (-1) ** l * sh.sh_block(l, r), atol=1e-13)
    assert np.allclose(sh.sh_block(l, 7.5 * r), sh.sh_block(l, r), atol=1e-13)


def test_quadrature_orthogonality():
    """(1/4pi) int Y_lm Y_l'm' dOmega = delta, Gauss-Legendre in cos(t) x uniform phi."""
    lmax = 4
    ct, wt = np.polynomial.legendre.leggauss(12)
    nphi = 16
    phi = 2 * np.pi * np.arange(nphi) / nphi
    C, F = np.meshgrid(ct, phi, indexing="ij")
    st = np.sqrt(1 - C**2)
    pts = np.stack([st * np.cos(F), st * np.sin(F), C], -1).reshape(-1, 3)
    wq = (wt[:, None] * np.full(nphi, 2 * np.pi / nphi)[None, :]).reshape(-1) / (4 * np.pi)
    Y = sh.sh(lmax, pts)
    G = (Y * wq[:, None]).T @ Y
    assert np.allclose(G, np.eye((lmax + 1) ** 2), atol=1e-12)


@pytest.mark.parametrize("lmax", [1, 3])
def test_gradient_by_central_differences(lmax):
    r = _dirs(25, 4)
    J = sh.sh_grad(lmax, r)
    h = 1e-6
    for a in range(3):
        d = np.zeros(3)
        d[a] = h
        fd = (sh.sh(lmax, r + d) - sh.sh(lmax, r - d)) / (2 * h)
        assert np.allclose(J[..., a], fd, atol=1e-7), a
    # the derivative is tangent: r . dY/dr = 0 (Y depends on the direction only)
    assert np.allclose(np.einsum("ekc,ec->ek", J, r), 0.0, atol=1e-12)


def test_degenerate_zero_vector():
    r = np.zeros((2, 3))
    r[1] = [1e-14, 0, 0]
    Y = sh.sh(3, r)
    assert np.all(Y[:, 0] == 1.0) and np.all(Y[:, 1:] == 0.0)
    assert np.all(sh.sh_grad(3, r) == 0.0)
