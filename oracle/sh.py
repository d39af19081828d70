"""Real spherical harmonics in FP64, written from their textbook definition.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may use anything under ``oracle/``.

Source passages. The pages name the operation but not its conventions:
  * "Machine Learning Interatomic Potentials: Advancing Open-Source Software for
    Efficient and Scalable Molecular Simulation", section "방법론 및 아키텍처",
    item 2 (e3j backend): the kernels target Clebsch-Gordan tensor products of
    MACE/NequIP, i.e. products of node irreps with spherical harmonics of the
    edge direction.
  * "High-performance training and inference for deep equivariant interatomic
    potentials", section "제안 방법": the Allegro tensor product contracts
    through Wigner 3-j coefficients.
No page prints a formula for Y_lm, so the readings below are this oracle's and
the GPU path's common contract:
  * component normalisation:  sum_m Y_lm(u)^2 = 2l+1 for every unit u;
  * no Condon-Shortley phase;  m ordered -l..l;
  * Y_lm = K_lm * (d^|m| P_l / dz^|m|)(z) * A_m(x, y), with
        K_lm = sqrt((2l+1) (l-|m|)! / (l+|m|)!) * (sqrt(2) if m != 0 else 1),
        A_m  = Re (x+iy)^m  (m > 0),  1 (m = 0),  Im (x+iy)^|m|  (m < 0).
    This is the usual P_l^|m|(cos t) * {cos, sin}(|m| phi) form, because on the
    unit sphere x + iy = sin(t) e^{i phi} and P_l^m(z) = (1-z^2)^{m/2} d^m P_l/dz^m.
  * Edge vectors shorter than 1e-12 give Y_0 = 1, Y_{l>=1} = 0 and a zero
    gradient (the degenerate direction).

The polynomial is kept as an explicit monomial table so that its gradient is an
exact polynomial derivative; the directional derivative with respect to the
unnormalised edge vector r is  dY/dr = (I - u u^T) grad_u P(u) / |r|.
"""
from __future__ import annotations

from functools import lru_cache
from math import comb, factorial, sqrt

import numpy as np

R_EPS = 1e-12  # below this length an edge has no direction


def legendre_coefficients(l: int) -> np.ndarray:
    """Coefficients a_k of P_l(z) = sum_k a_k z^k (explicit Legendre sum)."""
    a = np.zeros(l + 1)
    for k in range(l // 2 + 1):
        a[l - 2 * k] = (-1) ** k * comb(l, k) * comb(2 * l - 2 * k, l) / 2.0**l
    return a


def _differentiate(a: np.ndarray, times: int) -> np.ndarray:
    for _ in range(times):
        a = np.array([k * a[k] for k in range(1, len(a))]) if len(a) > 1 else np.zeros(1)
    return a


@lru_cache(maxsize=None)
def sh_monomials(l: int) -> tuple:
    """For m = -l..l, a tuple of {(px, py, pz): coeff} with Y_lm(u) = sum coeff x^px y^py z^pz."""
    out = []
    for m in range(-l, l + 1):
        mu = abs(m)
        zpoly = _differentiate(legendre_coefficients(l), mu)  # in z, degree l - mu
        norm = sqrt((2 * l + 1) * factorial(l - mu) / factorial(l + mu))
        if mu > 0:
            norm *= sqrt(2.0)
        # azimuthal factor: binomial expansion of (x + i y)^mu; i^k is real for even k
        az = {}
        for k in range(mu + 1):
            c = comb(mu, k)
            if m > 0 and k % 2 == 0:
                az[(mu - k, k)] = c * (-1) ** (k // 2)
            elif m < 0 and k % 2 == 1:
                az[(mu - k, k)] = c * (-1) ** ((k - 1) // 2)
        if m == 0:
            az = {(0, 0): 1.0}
        terms = {}
        for kz, cz in enumerate(zpoly):
            if cz == 0.0:
                continue
            for (px, py), ca in az.items():
                key = (px, py, kz)
                terms[key] = terms.get(key, 0.0) + norm * cz * ca
        out.append(terms)
    return tuple(out)


def _eval_poly(terms: dict, u: np.ndarray) -> np.ndarray:
    x, y, z = u[..., 0], u[..., 1], u[..., 2]
    acc = np.zeros(u.shape[:-1])
    for (px, py, pz), c in terms.items():
        acc = acc + c * x**px * y**py * z**pz
    return acc


def _eval_poly_grad(terms: dict, u: np.ndarray) -> np.ndarray:
    x, y, z = u[..., 0], u[..., 1], u[..., 2]
    g = np.zeros(u.shape)
    for (px, py, pz), c in terms.items():
        if px:
            g[..., 0] += c * px * x ** (px - 1) * y**py * z**pz
        if py:
            g[..., 1] += c * py * x**px * y ** (py - 1) * z**pz
        if pz:
            g[..., 2] += c * pz * x**px * y**py * z ** (pz - 1)
    return g


def _eval_poly_hess(terms: dict, u: np.ndarray) -> np.ndarray:
    """Second derivatives of the polynomial in u, shape [..., 3, 3]."""
    h = np.zeros(u.shape + (3,))
    for p, c in terms.items():
        for a in range(3):
            for b in range(3):
                q = list(p)
                f = q[a]
                q[a] -= 1
                if f == 0 or q[a] < 0:
                    continue
                f2 = q[b]
                q[b] -= 1
                if f2 == 0 or q[b] < 0:
                    continue
                h[..., a, b] += c * f * f2 * u[..., 0] ** q[0] * u[..., 1] ** q[1] * u[..., 2] ** q[2]
    return h


def sh_block(l: int, r: np.ndarray) -> np.ndarray:
    """Y_l(r/|r|), shape [..., 2l+1]."""
    r = np.asarray(r, dtype=np.float64)
    n = np.linalg.norm(r, axis=-1)
    ok = n >= R_EPS
    u = np.where(ok[..., None], r / np.where(ok, n, 1.0)[..., None], 0.0)
    vals = np.stack([_eval_poly(t, u) for t in sh_monomials(l)], axis=-1)
    if l > 0:
        vals[~ok] = 0.0
    else:
        vals[...] = 1.0
    return vals


def sh(lmax: int, r: np.ndarray) -> np.ndarray:
    """All blocks l = 0..lmax concatenated, shape [..., (lmax+1)^2]."""
    return np.concatenate([sh_block(l, r) for l in range(lmax + 1)], axis=-1)


def sh_grad(lmax: int, r: np.ndarray) -> np.ndarray:
    """dY_k/dr_a for the unnormalised vector r, shape [..., (lmax+1)^2, 3]."""
    r = np.asarray(r, dtype=np.float64)
    n = np.linalg.norm(r, axis=-1)
    ok = n >= R_EPS
    safe = np.where(ok, n, 1.0)
    u = np.where(ok[..., None], r / safe[..., None], 0.0)
    proj = np.eye(3) - u[..., :, None] * u[..., None, :]  # [..., 3, 3]
    blocks = []
    for l in range(lmax + 1):
        for t in sh_monomials(l):
            gu = _eval_poly_grad(t, u)  # [..., 3]
            d = np.einsum("...ab,...b->...a", proj, gu) / safe[..., None]
            d[~ok] = 0.0
            blocks.append(d)
    return np.stack(blocks, axis=-2)


def sh_hess(lmax: int, r: np.ndarray) -> np.ndarray:
    """d^2 Y_k / dr_a dr_b for the unnormalised vector r, shape [..., (lmax+1)^2, 3, 3].

    With u = r/n, n = |r|, P = I - u u^T, g = grad_u p(u) and K = the polynomial's
    second derivatives at u, the chain rule through u (du/dr = P / n) gives

        H = ( P K P - (u . g) P - u (P g)^T - (P g) u^T ) / n^2,

    symmetric in (a, b). Edges shorter than R_EPS give 0.
    """
    r = np.asarray(r, dtype=np.float64)
    n = np.linalg.norm(r, axis=-1)
    ok = n >= R_EPS
    safe = np.where(ok, n, 1.0)
    u = np.where(ok[..., None], r / safe[..., None], 0.0)
    proj = np.eye(3) - u[..., :, None] * u[..., None, :]
    blocks = []
    for l in range(lmax + 1):
        for t in sh_monomials(l):
            g = _eval_poly_grad(t, u)
            K = _eval_poly_hess(t, u)
            pg = np.einsum("...ab,...b->...a", proj, g)
            ug = np.einsum("...a,...a->...", u, g)
            H = (np.einsum("...ac,...cd,...db->...ab", proj, K, proj) - ug[..., None, None] * proj
                 - u[..., :, None] * pg[..., None, :] - pg[..., :, None] * u[..., None, :])
            H = H / (safe**2)[..., None, None]
            H[~ok] = 0.0
            blocks.append(H)
    return np.stack(blocks, axis=-3)
