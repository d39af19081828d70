"""FP64 oracle for the node-local product: equivariant features of higher correlation
order built from one node's own features, one weighted product per step.
TEST INFRASTRUCTURE ONLY (same rule as the rest of oracle/).

Passages: "FlashCart 如何让等变原子间势更快更准?", section "FlashCart 用笛卡尔内核替代球谐耦合"
(features are built recursively and brought back to a fixed width after every step,
which is what makes high correlation orders affordable) and section
"生成内核在高阶下胜过球谐基线" (the node-local product at 4096 nodes x 128 channels with
maximum rank 3 and 4; the forward of the path-reduced product is timed; the weighted
product is applied one step at a time and only ranks up to the chosen maximum are
kept after each step). The pages give no formula. The plain reading taken here:

  * B(1) = x, the node's features (ranks 0..L, C channels);
  * B(k+1)_l3[c] = sum over paths p = (l1, l2, l3) of w[k-1, p, c] * couple_p(B(k)_l1[c], x_l2[c]),
    for k = 1 .. K-1; the correlation order K is the number of factors of x in B(K);
  * the output is B(K); ranks above L are never formed (the path list stops at L),
    which is the "fixed width" of every step;
  * the channels do not mix; the weights w [K-1, P, C] are shared by all nodes;
  * the paths: l1, l2 and l3 each from the irreps 0..L, |l1 - l2| <= l3 <= l1 + l2,
    and, with parity letters, p1 * p2 == p3; ordered lexicographically by (l1, l2, l3);
  * couple_p is the spherical Clebsch-Gordan coupling (``cg.real_cg``, features in
    real spherical components) or the Cartesian coupling of STF tensors
    (``cartesian.couple``, features as full 3^l tensors).

The "full ladder" that the pages time beside the path-reduced product is named there
but not defined; it is not built.

Pinned by tests/test_oracle_nodelocal.py: order 1 is the identity, the scalar closed
form, closed forms of two-step ladders in both forms (which also fix the order in
which the steps take their weights), the Cartesian product against the spherical one
with per-path rescaled weights, and rotation equivariance.
"""
from __future__ import annotations

import numpy as np
import torch

from . import cartesian as ct
from . import cg as cg_mod
from . import paths as paths_mod


def node_paths(irreps: str):
    """The product's paths (l1, l2, l3): B's rank, x's rank, the result's rank."""
    ir = paths_mod.parse_irreps(irreps)
    use_parity = ir[0][1] is not None
    out = []
    for l1, p1 in ir:
        for l2, p2 in ir:
            for l3, p3 in ir:
                if not (abs(l1 - l2) <= l3 <= l1 + l2):
                    continue
                if use_parity and p1 * p2 != p3:
                    continue
                out.append((l1, l2, l3))
    return out


def _ranks(irreps: str):
    return [l for l, _ in paths_mod.parse_irreps(irreps)]


def _spherical_step(B: dict, X: dict, wk: np.ndarray, paths) -> dict:
    """One step in spherical components: blocks {l: [N, 2l+1, C]}, wk [P, C]."""
    new = {l: np.zeros_like(X[l]) for l in X}
    for p, (l1, l2, l3) in enumerate(paths):
        t = np.einsum("abm,nac,nbc->nmc", cg_mod.real_cg(l1, l2, l3), B[l1], X[l2])
        new[l3] += wk[p][None, None, :] * t
    return new


def node_product(x: np.ndarray, w: np.ndarray, irreps: str) -> np.ndarray:
    """Spherical node-local product. x [N, D, C] (rank blocks ascending, m = 0..2l in
    real spherical order), w [K-1, P, C]; returns B(K) [N, D, C]."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    paths = node_paths(irreps)
    assert w.ndim == 3 and w.shape[1] == len(paths) and w.shape[2] == x.shape[2], (w.shape, len(paths))
    X = {l: x[:, l * l:(l + 1) ** 2, :] for l in _ranks(irreps)}
    B = dict(X)
    for k in range(w.shape[0]):
        B = _spherical_step(B, X, w[k], paths)
    return np.concatenate([B[l] for l in _ranks(irreps)], axis=1)


def _cartesian_step(B: dict, X: dict, wk: torch.Tensor, paths, C: int) -> dict:
    """One step on full STF tensors {l: [N, C] + [3] * l}, wk [P, C]."""
    new = {l: torch.zeros_like(X[l]) for l in X}
    for p, (l1, l2, l3) in enumerate(paths):
        t = ct.couple(B[l1], X[l2], l1, l2, l3)
        new[l3] = new[l3] + t * wk[p].reshape(1, C, *([1] * l3))
    return new


def node_product_cartesian(x: dict, w, irreps: str) -> dict:
    """Cartesian node-local product. x {l: [N, C] + [3] * l} STF tensors, w [K-1, P, C];
    returns B(K) in the same form."""
    w = torch.as_tensor(np.asarray(w), dtype=torch.float64)
    paths = node_paths(irreps)
    C = w.shape[2]
    assert w.shape[1] == len(paths), (w.shape, len(paths))
    X = {l: torch.as_tensor(x[l], dtype=torch.float64) for l in _ranks(irreps)}
    B = dict(X)
    for k in range(w.shape[0]):
        B = _cartesian_step(B, X, w[k], paths, C)
    return B
