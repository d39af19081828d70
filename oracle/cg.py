"""Real Clebsch-Gordan coupling tensors in FP64 by invariance (null-space) construction.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source passages:
  * "High-performance training and inference for deep equivariant interatomic
    potentials", section "제안 방법": the tensor product contracts through
    Wigner 3-j coefficients, stored sparsely (compressed sparse format).
  * "Machine Learning Interatomic Potentials: Advancing Open-Source Software ...",
    section "방법론 및 아키텍처", item 2: Clebsch-Gordan tensor products.
The pages print no coefficient, so the tensor is fixed by what it must do:

  * CG^{(l1 l2 l3)}[m1, m2, m3] is the (unique up to scale, for the SO(3) triangle
    rule |l1-l2| <= l3 <= l1+l2) real tensor that makes
        out_m3 = sum_{m1, m2} CG[m1, m2, m3] x_m1 y_m2
    rotate as an l3 irrep whenever x, y rotate as l1, l2 irreps in the real
    spherical-harmonic basis of ``oracle/sh.py``;
  * normalisation: sum_{m1, m2} CG[m1, m2, m3]^2 = 1 for every m3;
  * sign: the first nonzero entry in lexicographic (m1, m2, m3) order (indices
    0..2l) is positive;
  * entries below 1e-13 in magnitude are exact zeros (the sparsity pattern).

Construction: the rotation matrices D^l(R) of the basis are fitted from the
harmonics themselves, D^l = Y_l(R r_k) pinv(Y_l(r_k)) over 4(2l+1) random
directions r_k; the coupling M (shape d3 x d1 d2, out = M (x kron y)) solves
M kron(D1, D2) = D3 M for two random rotations at once (their common fixed space
is the invariant space), taken as the right null space of the stacked system.
"""
from __future__ import annotations

from functools import lru_cache

import numpy as np

from . import sh as _sh

ZERO_TOL = 1e-13


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    """A uniformly random proper rotation (QR of a Gaussian matrix, sign-fixed)."""
    q, r = np.linalg.qr(rng.standard_normal((3, 3)))
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


def wigner_d(l: int, R: np.ndarray, seed: int = 12345) -> np.ndarray:
    """D^l(R) with Y_l(R r) = D^l(R) Y_l(r) for the basis of ``oracle/sh.py``."""
    rng = np.random.default_rng(seed + 97 * l)
    pts = rng.standard_normal((4 * (2 * l + 1), 3))
    pts /= np.linalg.norm(pts, axis=1, keepdims=True)
    A = _sh.sh_block(l, pts)            # [n, d]
    B = _sh.sh_block(l, pts @ R.T)      # [n, d], rows Y(R p)
    # B^T = D A^T  =>  D = B^T pinv(A^T)
    return B.T @ np.linalg.pinv(A.T)


def triangle(l1: int, l2: int, l3: int) -> bool:
    return abs(l1 - l2) <= l3 <= l1 + l2


@lru_cache(maxsize=None)
def real_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    """CG[m1, m2, m3] (shape [2l1+1, 2l2+1, 2l3+1]); all zeros off the triangle rule."""
    d1, d2, d3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    if not triangle(l1, l2, l3):
        return np.zeros((d1, d2, d3))
    rng = np.random.default_rng(2024 + 100 * l1 + 10 * l2 + l3)
    rows = []
    for _ in range(2):
        R = random_rotation(rng)
        D1, D2, D3 = wigner_d(l1, R), wigner_d(l2, R), wigner_d(l3, R)
        K = np.kron(D1, D2)
        # row-major vec: vec(M K) = (I kron K^T) vec(M), vec(D3 M) = (D3 kron I) vec(M)
        rows.append(np.kron(np.eye(d3), K.T) - np.kron(D3, np.eye(d1 * d2)))
    A = np.concatenate(rows, axis=0)
    _, s, vt = np.linalg.svd(A)
    null_dim = int(np.sum(s < 1e-9))
    if null_dim != 1:
        raise AssertionError(f"invariant space of ({l1},{l2},{l3}) has dim {null_dim}")
    M = vt[-1].reshape(d3, d1 * d2)
    cg = M.reshape(d3, d1, d2).transpose(1, 2, 0).copy()
    col = np.sum(cg**2, axis=(0, 1))      # Schur: equal for every m3
    if np.max(np.abs(col - col.mean())) > 1e-10 * col.mean():
        raise AssertionError("coupling is not an isometry in (m1, m2)")
    cg /= np.sqrt(col.mean())
    cg[np.abs(cg) < ZERO_TOL] = 0.0
    flat = cg.reshape(-1)
    first = flat[np.flatnonzero(flat)[0]]
    if first < 0:
        cg = -cg
    return cg + 0.0  # no negative zeros


def nnz_list(l1: int, l2: int, l3: int):
    """Sparse form: list of (m1, m2, m3, value) with indices 0..2l, lexicographic."""
    cg = real_cg(l1, l2, l3)
    idx = np.argwhere(cg != 0.0)
    return [(int(a), int(b), int(c), float(cg[a, b, c])) for a, b, c in idx]
