"""Pins of the library's edge-frame tables (generated at build time by
csrc/gen_tables.cpp) against the oracle's independent constructions.

The kernels evaluate the tensor product in a frame where the edge lies on z:
  CG_p(x, Y(u)) = D_l3(R)^T B_p D_l1(R) x  with R u = z,
so they need B_p (the m2 = 0 slice of each coupling times sqrt(2 l2 + 1)), the
rotation generators J_x, J_y (for the derivative with respect to the edge
direction) and the matrices that fit D_l(R) from harmonics at 7 fixed points.
Each table is checked here against the oracle's coupling tensors, its
harmonics and its Wigner matrices (fitted from harmonics, a different
construction from the library's ladder-operator and Racah formulas).
"""
import os
import re

import numpy as np
import pytest

from cg_tensor_products_b200 import build as etp_build
from oracle import cg, sh

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "cg_tensor_products_b200", "csrc", "generated", "etp_tables.h")


def _array(txt, name, shape):
    body = re.split(rf"constexpr double {name}\[[^=]*= {{", txt)[1].split("};", 1)[0]
    vals = [float(v) for v in re.findall(r"-?\d+(?:\.\d+)?(?:[eE][-+]?\d+)?", body)]
    return np.array(vals).reshape(shape)


@pytest.fixture(scope="module")
def tables():
    etp_build.build()
    with open(HEADER) as f:
        txt = f.read()
    return {"B": _array(txt, "kFrameB", (4, 4, 4, 4)), "J": _array(txt, "kGen", (2, 4, 7, 7)),
            "P": _array(txt, "kFitPoints", (7, 3)), "Ainv": _array(txt, "kFitInv", (4, 7, 7))}


def test_frame_coupling_slices(tables):
    for l1 in range(4):
        for l2 in range(4):
            for l3 in range(4):
                full = np.sqrt(2 * l2 + 1) * cg.real_cg(l1, l2, l3)[:, l2, :]   # [m1, m3]
                want = np.zeros_like(full)
                odd = (l1 + l2 + l3) % 2 == 1
                for mu in range(min(l1, l3) + 1):
                    b = tables["B"][l1, l2, l3, mu]
                    if odd:
                        if mu:
                            want[l1 - mu, l3 + mu] = b
                            want[l1 + mu, l3 - mu] = -b
                    else:
                        want[l1 + mu, l3 + mu] = b
                        want[l1 - mu, l3 - mu] = b
                assert np.max(np.abs(want - full)) < 1e-12, (l1, l2, l3)


def test_generators_against_differentiated_wigner_matrices(tables):
    from scipy.spatial.transform import Rotation

    eps = 1e-5
    for axis in (0, 1):
        v = np.zeros(3)
        v[axis] = eps
        Rp, Rm = Rotation.from_rotvec(v).as_matrix(), Rotation.from_rotvec(-v).as_matrix()
        for l in range(4):
            d = 2 * l + 1
            fd = (cg.wigner_d(l, Rp) - cg.wigner_d(l, Rm)) / (2 * eps)
            assert np.max(np.abs(tables["J"][axis, l, :d, :d] - fd)) < 1e-8, (axis, l)


def test_fitted_wigner_matrices(tables):
    P, Ainv = tables["P"], tables["Ainv"]
    assert np.allclose(np.linalg.norm(P, axis=1), 1.0, atol=1e-15)
    rng = np.random.default_rng(0)
    for _ in range(5):
        R = cg.random_rotation(rng)
        for l in (2, 3):
            d = 2 * l + 1
            Yr = sh.sh_block(l, P[:d] @ R.T).T           # columns Y_l(R p_k)
            assert np.max(np.abs(Yr @ Ainv[l, :d, :d] - cg.wigner_d(l, R))) < 1e-12, l
