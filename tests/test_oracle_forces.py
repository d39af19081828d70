"""Pins of the FP64 force / virial assembly (oracle/forces.py) against what the
mathematics fixes: a one-edge closed form, momentum conservation, and central
finite differences of an energy with respect to atom positions and to a
homogeneous strain (the energy is the oracle's tensor product contracted with a
fixed cotangent, so it depends on positions only through the edge vectors)."""
import numpy as np
import pytest

import oracle
import workloads


def _system(seed, n=9, e=40, L=2, C=3):
    rng = np.random.default_rng(seed)
    pos = rng.normal(0.0, 1.5, (n, 3))
    dst = rng.integers(0, n, e)
    src = (dst + rng.integers(1, n, e)) % n          # no self-loops
    row_ptr, s, order = workloads.csr_from_pairs(n, dst, src)
    d_sorted = dst[order]
    D, P = (L + 1) ** 2, 15 if L == 2 else 5
    x = rng.normal(size=(n, D, C))
    w = rng.normal(size=(e, P, C)) / np.sqrt(P)
    G = rng.normal(size=(n, D, C))
    tp = oracle.OracleTP(f"0..{L}", L, f"0..{L}", C)
    return pos, row_ptr, s, d_sorted, x, w, G, tp


def _energy(pos, row_ptr, s, d, x, w, G, tp):
    r = pos[s] - pos[d]
    return float(np.sum(tp.forward(row_ptr, s, r, x, w) * G))


@pytest.fixture(scope="module", autouse=True)
def _built():
    oracle.build()


def test_single_edge_closed_form():
    row_ptr = np.array([0, 1, 1], np.int32)        # node 0 receives one edge from node 1
    src = np.array([1], np.int32)
    r = np.array([[0.3, -1.2, 2.0]])
    g = np.array([[1.5, 0.25, -0.75]])
    F, V = oracle.assemble_forces(2, row_ptr, src, r, g)
    assert np.array_equal(F, np.array([g[0], -g[0]]))
    assert np.array_equal(V[0], np.outer(g[0], r[0])) and np.array_equal(V[1], np.zeros((3, 3)))


def test_momentum_conservation():
    rng = np.random.default_rng(3)
    wl = workloads.random_graph(rng, 50, 700, 1, 4, 5)
    g = rng.normal(size=(wl.E, 3))
    F, _ = oracle.assemble_forces(wl.N, wl.row_ptr, wl.src, wl.r, g)
    assert np.abs(F.sum(axis=0)).max() < 1e-12 * np.abs(g).sum()


@pytest.mark.parametrize("seed", [0, 1])
def test_forces_are_minus_the_position_gradient(seed):
    pos, row_ptr, s, d, x, w, G, tp = _system(seed)
    r = pos[s] - pos[d]
    grad_r = tp.backward(row_ptr, s, r, x, w, G, want=("r",))["grad_r"]
    F, _ = oracle.assemble_forces(len(pos), row_ptr, s, r, grad_r)
    h = 1e-6
    fd = np.zeros_like(pos)
    for k in range(len(pos)):
        for a in range(3):
            p1, p0 = pos.copy(), pos.copy()
            p1[k, a] += h
            p0[k, a] -= h
            fd[k, a] = -(_energy(p1, row_ptr, s, d, x, w, G, tp) - _energy(p0, row_ptr, s, d, x, w, G, tp)) / (2 * h)
    assert np.abs(F - fd).max() < 1e-7 * max(1.0, np.abs(fd).max())


def test_virial_is_the_strain_derivative():
    pos, row_ptr, s, d, x, w, G, tp = _system(5)
    r = pos[s] - pos[d]
    grad_r = tp.backward(row_ptr, s, r, x, w, G, want=("r",))["grad_r"]
    _, V = oracle.assemble_forces(len(pos), row_ptr, s, r, grad_r)
    total = V.sum(axis=0)
    h = 1e-6
    fd = np.zeros((3, 3))
    for a in range(3):
        for b in range(3):
            eps = np.zeros((3, 3))
            eps[a, b] = h
            ep = _energy(pos @ (np.eye(3) + eps).T, row_ptr, s, d, x, w, G, tp)
            em = _energy(pos @ (np.eye(3) - eps).T, row_ptr, s, d, x, w, G, tp)
            fd[a, b] = (ep - em) / (2 * h)
    assert np.abs(total - fd).max() < 1e-7 * max(1.0, np.abs(fd).max())
    assert np.abs(total - total.T).max() > 1e-3      # not symmetric here: the (a, b) order is pinned


def test_planted_mistakes_are_caught():
    """A swapped destination/source, or the virial transposed, fails the pins above."""
    pos, row_ptr, s, d, x, w, G, tp = _system(0)
    r = pos[s] - pos[d]
    grad_r = tp.backward(row_ptr, s, r, x, w, G, want=("r",))["grad_r"]
    F, V = oracle.assemble_forces(len(pos), row_ptr, s, r, grad_r)
    k, a, h = 2, 1, 1e-6
    p1, p0 = pos.copy(), pos.copy()
    p1[k, a] += h
    p0[k, a] -= h
    fd = -(_energy(p1, row_ptr, s, d, x, w, G, tp) - _energy(p0, row_ptr, s, d, x, w, G, tp)) / (2 * h)
    swapped = np.zeros_like(F)
    np.add.at(swapped, s, grad_r)
    np.add.at(swapped, d, -grad_r)
    assert abs(F[k, a] - fd) < 1e-7 * max(1.0, abs(fd)) and abs(swapped[k, a] - fd) > 1e-3
    tot = V.sum(axis=0)
    assert np.abs(tot - tot.T).max() > 1e-3
