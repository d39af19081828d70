"""FP64 oracle for the radial weights of an edge: a small MLP of the edge length.
TEST INFRASTRUCTURE ONLY (same rule as the rest of oracle/).

Interatomic potentials of the pages' kind make the per-edge, per-path,
per-channel weights w of the tensor product a learned function of the edge
length ("High-performance training and inference for deep equivariant
interatomic potentials", section "제안 방법": the Allegro tensor product and its
fused kernels; the water systems of section "주요 결과" are evaluated with such a
model). The plain reading taken here, with d = |r_e| and cutoff r_c:

    b_n(d) = sqrt(2 / r_c) sin(n pi d / r_c) / d,   n = 1 .. n_basis   (Bessel basis, no envelope)
    z = b W1,  h = SiLU(z) = z / (1 + exp(-z)),  w = h W2   (no biases)

with W1 [n_basis, hidden], W2 [hidden, P*C] and w reshaped to [P, C]. At d = 0
the basis takes its limit sqrt(2 / r_c) n pi / r_c and its derivative is taken
as 0 (an edge of zero length has no direction either).

The vector-Jacobian product for a cotangent G = dL/dw:

    grad_W2 = sum_e h_e^T G_e,   dL/dh = G W2^T,   dL/dz = dL/dh * SiLU'(z),
    grad_W1 = sum_e b_e^T dL/dz_e,   dL/dd = (dL/dz W1^T) . db/dd,
    grad_r (through d) = dL/dd * r / |r|.
"""
from __future__ import annotations

import numpy as np

D_EPS = 1e-12


def bessel(d: np.ndarray, rc: float, n_basis: int):
    """(b [E, n_basis], db/dd [E, n_basis]) in float64."""
    d = np.asarray(d, dtype=np.float64)
    n = np.arange(1, n_basis + 1, dtype=np.float64)[None, :]
    k = n * np.pi / rc
    c = np.sqrt(2.0 / rc)
    small = d < D_EPS
    ds = np.where(small, 1.0, d)[:, None]
    b = c * np.sin(k * ds) / ds
    db = c * (k * np.cos(k * ds) / ds - np.sin(k * ds) / ds**2)
    b = np.where(small[:, None], c * k, b)
    db = np.where(small[:, None], 0.0, db)
    return b, db


def silu(z):
    return z / (1.0 + np.exp(-z))


def silu_grad(z):
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


class RadialMLP:
    """w(r) = SiLU(bessel(|r|) W1) W2, reshaped to [E, P, C]."""

    def __init__(self, W1: np.ndarray, W2: np.ndarray, rc: float, P: int, C: int):
        self.W1 = np.asarray(W1, dtype=np.float64)
        self.W2 = np.asarray(W2, dtype=np.float64)
        self.rc, self.P, self.C = float(rc), int(P), int(C)
        assert self.W2.shape == (self.W1.shape[1], self.P * self.C)

    def _hidden(self, r):
        r = np.asarray(r, dtype=np.float64)
        d = np.linalg.norm(r, axis=1)
        b, db = bessel(d, self.rc, self.W1.shape[0])
        z = b @ self.W1
        return r, d, b, db, z

    def forward(self, r) -> np.ndarray:
        _, _, _, _, z = self._hidden(r)
        return (silu(z) @ self.W2).reshape(len(z), self.P, self.C)

    def backward(self, r, grad_w) -> dict:
        """grad_W1 [n_basis, hidden], grad_W2 [hidden, P*C], grad_r [E, 3] (through |r| only)."""
        r, d, b, db, z = self._hidden(r)
        G = np.asarray(grad_w, dtype=np.float64).reshape(len(z), -1)
        h = silu(z)
        grad_W2 = h.T @ G
        gz = (G @ self.W2.T) * silu_grad(z)
        grad_W1 = b.T @ gz
        dd = np.sum((gz @ self.W1.T) * db, axis=1)
        unit = np.where(d[:, None] < D_EPS, 0.0, r / np.where(d < D_EPS, 1.0, d)[:, None])
        return {"grad_W1": grad_W1, "grad_W2": grad_W2, "grad_r": dd[:, None] * unit}
