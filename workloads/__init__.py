"""Seeded synthetic inputs for the edge tensor product: graphs, edge vectors, features, weights.

This module serves both the CUDA path (tests, bench, smoke) and the oracle. It
holds none of the method's arithmetic: it builds CSR-by-destination neighbour
graphs, draws the edge vectors, node features x, per-edge weights w and the
cotangent g, and nothing else. The numbers of paths per workload are stated
here as data (5, 15, 34 for the SO(3) path set at L = 1, 2, 3).

Workloads (each stands in for a workload the pages describe; no dataset exists
or is needed):
  tiny      32 nodes uniform in a periodic 6 A box, 8 nearest neighbours each
            (minimum image; ties by node id), L=1, C=8.
  micro_l2  1024 nodes x exactly 128 distinct neighbours drawn uniformly without
            self-loops; edge vectors ~ 2 N(0, I3) A; L=2, C=128. Shape of the
            edge-convolution micro-benchmark in "FlashCart 如何让等变原子间势更快
            更准?", section "生成内核在高阶下胜过球谐基线" (1024 nodes, 128
            channels, 128 neighbours).
  micro_l3  the same graph and edge vectors (same seed), L=3, C=128.
  water     1024 H2O at 1 g/cm^3 (box 31.29 A), O uniform, H at 0.96 A and 104.5
            deg in a random orientation, every atom jittered N(0, 0.1 A); periodic
            radius graph r < 5 A; L=2, C=64; w from a seeded radial MLP of |r|
            (8 Bessel functions, hidden 64, SiLU) evaluated in FP64 on the CPU.
            Water boxes are the small-system MD workload of "High-performance
            training and inference for deep equivariant interatomic potentials",
            section "주요 결과".
  large     32768 atoms uniform at 0.1 / A^3 (box 68.95 A), periodic radius graph
            r < 4.5 A (~38 neighbours per atom), node ids randomly permuted after
            the graph is built; L=3, C=64. Stands in for the large systems of
            "Scaling the leading accuracy of deep equivariant models to
            biomolecular simulations of realistic size".

Draw order from numpy.random.default_rng(seed): geometry, edge vectors (micro
only), x, w (or the MLP parameters), g. Every row of a CSR lists its sources in
ascending order; edges are directed i <- j with r_e = pos[j] - pos[i] under the
minimum-image convention.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

N_PATHS_SO3 = {0: 1, 1: 5, 2: 15, 3: 34}


@dataclass
class Workload:
    name: str
    L: int
    C: int
    P: int
    row_ptr: np.ndarray   # int32 [N+1]
    src: np.ndarray       # int32 [E]
    r: np.ndarray         # float32 [E, 3]
    x: np.ndarray         # float32 [N, (L+1)^2, C]
    w: np.ndarray         # float32 [E, P, C]
    g: np.ndarray         # float32 [N, (L+1)^2, C]
    # the radial MLP that produced w (water only): W1 [8, 64], W2 [64, P*C] float32, cutoff
    W1: np.ndarray | None = None
    W2: np.ndarray | None = None
    r_cut: float | None = None
    # atom positions in the periodic box, float32 [N, 3], and the radius-graph cutoff (water, large)
    pos: np.ndarray | None = None
    graph_cutoff: float | None = None

    @property
    def N(self) -> int:
        return len(self.row_ptr) - 1

    @property
    def E(self) -> int:
        return len(self.src)

    @property
    def irreps(self) -> str:
        return f"0..{self.L}"


SPECS = {
    "tiny": dict(L=1, C=8),
    "micro_l2": dict(L=2, C=128),
    "micro_l3": dict(L=3, C=128),
    "water": dict(L=2, C=64),
    "large": dict(L=3, C=64),
}


def csr_from_pairs(n: int, dst: np.ndarray, src: np.ndarray):
    """Sort directed edges by (dst, src) and return row_ptr, src, and the sort order."""
    order = np.lexsort((src, dst))
    counts = np.bincount(dst, minlength=n)
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return row_ptr, src[order].astype(np.int32), order


def min_image(d: np.ndarray, box: float) -> np.ndarray:
    return d - box * np.round(d / box)


def radius_pairs(pos: np.ndarray, box: float, rc: float):
    """All ordered pairs (i, j), i != j, with minimum-image distance strictly below rc."""
    from scipy.spatial import cKDTree

    pos = np.mod(pos, box)
    tree = cKDTree(pos, boxsize=box)
    pairs = tree.query_pairs(rc * (1 + 1e-9), output_type="ndarray")
    i, j = pairs[:, 0], pairs[:, 1]
    d = np.linalg.norm(min_image(pos[j] - pos[i], box), axis=1)
    keep = d < rc
    i, j = i[keep], j[keep]
    return np.concatenate([i, j]), np.concatenate([j, i])


def _normal(rng, shape, scale=None):
    a = rng.standard_normal(shape, dtype=np.float32)
    if scale is not None:
        a *= np.float32(scale)
    return a


def _geometry_tiny(rng):
    n, box, k = 32, 6.0, 8
    pos = rng.uniform(0.0, box, size=(n, 3))
    dst, src = [], []
    for i in range(n):
        d = np.linalg.norm(min_image(pos - pos[i], box), axis=1)
        cand = [(d[j], j) for j in range(n) if j != i]
        cand.sort()
        for _, j in cand[:k]:
            dst.append(i)
            src.append(j)
    dst, src = np.array(dst), np.array(src)
    row_ptr, src_sorted, order = csr_from_pairs(n, dst, src)
    dst_sorted = dst[order]
    r = min_image(pos[src_sorted] - pos[dst_sorted], box)
    return row_ptr, src_sorted, r.astype(np.float32)


def _geometry_micro(rng, n=1024):
    k = 128
    dst = np.repeat(np.arange(n), k)
    src = np.empty(n * k, dtype=np.int64)
    for i in range(n):
        c = rng.choice(n - 1, size=k, replace=False)
        c = c + (c >= i)
        src[i * k:(i + 1) * k] = np.sort(c)
    row_ptr = np.arange(0, n * k + 1, k, dtype=np.int32)
    r = _normal(rng, (n * k, 3), 2.0)
    return row_ptr, src.astype(np.int32), r


def water_box_side(n_mol: int = 1024) -> float:
    grams = n_mol * 18.015 / 6.02214076e23
    return (grams / 1.0) ** (1.0 / 3.0) * 1e8  # cm -> A at 1 g/cm^3


def _random_rotations(rng, n):
    q = rng.standard_normal((n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    a, b, c, d = q.T
    return np.stack([
        np.stack([a*a + b*b - c*c - d*d, 2*(b*c - a*d), 2*(b*d + a*c)], -1),
        np.stack([2*(b*c + a*d), a*a - b*b + c*c - d*d, 2*(c*d - a*b)], -1),
        np.stack([2*(b*d - a*c), 2*(c*d + a*b), a*a - b*b - c*c + d*d], -1),
    ], -2)


def _geometry_water(rng, rc=5.0):
    n_mol = 1024
    box = water_box_side(n_mol)
    o = rng.uniform(0.0, box, size=(n_mol, 3))
    half = np.deg2rad(104.5) / 2
    local = 0.96 * np.array([[np.sin(half), 0.0, np.cos(half)],
                             [-np.sin(half), 0.0, np.cos(half)]])
    rot = _random_rotations(rng, n_mol)
    h = o[:, None, :] + np.einsum("nab,kb->nka", rot, local)
    pos = np.concatenate([o[:, None, :], h], axis=1).reshape(-1, 3)
    pos = pos + rng.normal(0.0, 0.1, size=pos.shape)
    pos = np.mod(pos, box)
    n = len(pos)
    dst, src = radius_pairs(pos, box, rc)
    row_ptr, src_sorted, order = csr_from_pairs(n, dst, src)
    r = min_image(pos[src_sorted] - pos[dst[order]], box)
    return row_ptr, src_sorted, r, rc, pos


def _geometry_large(rng, rc=4.5, n=32768):
    dens = 0.1
    box = (n / dens) ** (1.0 / 3.0)
    pos = rng.uniform(0.0, box, size=(n, 3))
    dst, src = radius_pairs(pos, box, rc)
    rvec = min_image(pos[src] - pos[dst], box)
    perm = rng.permutation(n)             # old id -> new id
    dst, src = perm[dst], perm[src]
    row_ptr, src_sorted, order = csr_from_pairs(n, dst, src)
    pos_new = np.empty_like(pos)
    pos_new[perm] = pos
    return row_ptr, src_sorted, rvec[order], rc, pos_new


def radial_mlp_weights(rng, r: np.ndarray, rc: float, P: int, C: int,
                       n_basis: int = 8, hidden: int = 64):
    """(w, W1, W2): w[e] = Linear(64 -> P*C)(SiLU(Linear(8 -> 64)(bessel(|r_e|)))) in FP64, cast to
    fp32, and the MLP's weights W1 [8, 64], W2 [64, P*C] cast to fp32.

    Bessel basis b_n(d) = sqrt(2/rc) sin(n pi d / rc) / d, n = 1..8, no envelope;
    weights N(0, 1/fan_in), no biases.
    """
    W1 = rng.standard_normal((n_basis, hidden)) / np.sqrt(n_basis)
    W2 = rng.standard_normal((hidden, P * C)) / np.sqrt(hidden)
    d = np.linalg.norm(r.astype(np.float64), axis=1)
    n = np.arange(1, n_basis + 1)
    b = np.sqrt(2.0 / rc) * np.sin(n[None, :] * np.pi * d[:, None] / rc) / d[:, None]
    h = b @ W1
    h = h / (1.0 + np.exp(-h))
    out = np.empty((len(d), P * C), dtype=np.float32)
    step = 16384
    for s in range(0, len(d), step):
        out[s:s + step] = (h[s:s + step] @ W2).astype(np.float32)
    return out.reshape(len(d), P, C), W1.astype(np.float32), W2.astype(np.float32)


def make(name: str, seed: int = 0, n_nodes: int | None = None) -> Workload:
    """Build one named workload from numpy.random.default_rng(seed).

    n_nodes (micro and large workloads) shrinks the node count: micro keeps 128
    neighbours per node, large keeps its density and cutoff (about 38 neighbours);
    profiling captures use it to stay small."""
    spec = SPECS[name]
    L, C = spec["L"], spec["C"]
    P = N_PATHS_SO3[L]
    D = (L + 1) ** 2
    rng = np.random.default_rng(seed)
    if name == "tiny":
        row_ptr, src, r = _geometry_tiny(rng)
    elif name in ("micro_l2", "micro_l3"):
        row_ptr, src, r = _geometry_micro(rng, n_nodes or 1024)
    elif name == "water":
        row_ptr, src, r64, rc, pos = _geometry_water(rng)
        r = r64.astype(np.float32)
    elif name == "large":
        row_ptr, src, r64, rc, pos = _geometry_large(rng, n=n_nodes or 32768)
        r = r64.astype(np.float32)
    else:
        raise KeyError(name)
    N, E = len(row_ptr) - 1, len(src)
    x = _normal(rng, (N, D, C))
    mlp = {}
    if name == "water":
        w, W1, W2 = radial_mlp_weights(rng, r64, rc, P, C)
        mlp = dict(W1=W1, W2=W2, r_cut=rc)
    else:
        w = _normal(rng, (E, P, C), 1.0 / np.sqrt(P))
    g = _normal(rng, (N, D, C))
    geo = dict(pos=pos.astype(np.float32), graph_cutoff=rc) if name in ("water", "large") else {}
    return Workload(name, L, C, P, row_ptr, src.astype(np.int32), np.ascontiguousarray(r), x, w, g, **mlp, **geo)


def random_graph(rng, n: int, e: int, L: int, C: int, P: int, empty_rows=True) -> Workload:
    """A small ragged random multigraph (duplicates and empty rows allowed) for edge cases."""
    dst = rng.integers(0, n, size=e)
    if empty_rows and n > 2:
        dst = np.where(dst == n // 2, (n // 2 + 1) % n, dst)   # node n//2 has no incoming edge
    src = rng.integers(0, n, size=e)
    if empty_rows and n > 3:
        src = np.where(src == n // 3, (n // 3 + 2) % n, src)   # node n//3 has no outgoing edge
    row_ptr, src_sorted, order = csr_from_pairs(n, dst, src)
    D = (L + 1) ** 2
    r = _normal(rng, (e, 3), 1.5)
    x = _normal(rng, (n, D, C))
    w = _normal(rng, (e, P, C), 1.0 / np.sqrt(P))
    g = _normal(rng, (n, D, C))
    return Workload("random", L, C, P, row_ptr, src_sorted, r, x, w, g)
