"""FP64 oracle for assembling atom forces and per-atom virials from per-edge
energy derivatives. TEST INFRASTRUCTURE ONLY (same rule as the rest of oracle/).

The pages evaluate models on energies and forces ("FlashCart 如何让等变原子间势更快更准?",
section "560 万参数模型胜过 1.89 亿参数 transformer": energy and force errors and the time
to evaluate energy and forces per atom). Forces are the negative position gradient
of the energy; when the energy depends on positions only through the edge vectors
r_e = pos[src e] - pos[dst e] (plus a fixed periodic shift), the chain rule gives,
with g_e = dE/dr_e,

    F_k = -dE/dpos_k = sum_{e: dst e = k} g_e - sum_{e: src e = k} g_e,

and under a homogeneous strain of every edge vector r -> (I + eps) r,

    dE/d eps_ab = sum_e g_e[a] r_e[b],

which this module splits per atom by giving each edge's term to its destination:
virial[k, a, b] = sum_{e: dst e = k} g_e[a] r_e[b].

Written as the definition's plain loops over edges (numpy's unbuffered add.at).
"""
from __future__ import annotations

import numpy as np


def assemble_forces(n_nodes: int, row_ptr: np.ndarray, src: np.ndarray, r: np.ndarray, grad_r: np.ndarray):
    """(forces [N, 3], virial [N, 3, 3]) in float64 from g = grad_r [E, 3]."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    src = np.asarray(src, dtype=np.int64)
    g = np.asarray(grad_r, dtype=np.float64)
    rr = np.asarray(r, dtype=np.float64)
    E = len(src)
    dst = np.repeat(np.arange(n_nodes), np.diff(row_ptr))
    assert len(dst) == E and g.shape == (E, 3) and rr.shape == (E, 3)
    forces = np.zeros((n_nodes, 3))
    np.add.at(forces, dst, g)
    np.add.at(forces, src, -g)
    virial = np.zeros((n_nodes, 3, 3))
    np.add.at(virial, dst, g[:, :, None] * rr[:, None, :])
    return forces, virial
