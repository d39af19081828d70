"""Pins of the FP64 radial-weight MLP (oracle/radial.py): closed forms of the
Bessel basis and SiLU, central differences of its vector-Jacobian product, a
planted mistake, and the whole chain (radial weights -> tensor product ->
energy -> forces) against finite differences in the atom positions."""
import numpy as np
import pytest

import oracle
import workloads
from oracle import radial


def test_bessel_closed_forms():
    rc, nb = 5.0, 8
    n = np.arange(1, nb + 1)
    c = np.sqrt(2 / rc)
    b, db = radial.bessel(np.array([rc, rc / 2, 0.0]), rc, nb)
    assert np.abs(b[0]).max() < 1e-15                                   # sin(n pi) = 0 at the cutoff
    assert np.allclose(b[1], c * np.sin(n * np.pi / 2) / (rc / 2), atol=1e-15)
    assert np.allclose(b[2], c * n * np.pi / rc) and np.all(db[2] == 0)  # the d -> 0 limit
    d = np.array([0.7, 2.3, 4.9])
    h = 1e-6
    fd = (radial.bessel(d + h, rc, nb)[0] - radial.bessel(d - h, rc, nb)[0]) / (2 * h)
    assert np.abs(fd - radial.bessel(d, rc, nb)[1]).max() < 1e-8


def test_silu_closed_forms():
    assert radial.silu(0.0) == 0.0 and radial.silu_grad(0.0) == 0.5
    z = np.linspace(-6, 6, 25)
    assert np.allclose(radial.silu(z), z * 0.5 * (1 + np.tanh(z / 2)), atol=1e-15)
    h = 1e-6
    assert np.abs((radial.silu(z + h) - radial.silu(z - h)) / (2 * h) - radial.silu_grad(z)).max() < 1e-9


def _mlp(seed, P=5, C=3, nb=8, hidden=6, rc=5.0):
    rng = np.random.default_rng(seed)
    return radial.RadialMLP(rng.normal(size=(nb, hidden)) / np.sqrt(nb), rng.normal(size=(hidden, P * C)) / np.sqrt(hidden),
                            rc, P, C), rng


def test_vjp_matches_central_differences():
    mlp, rng = _mlp(1)
    r = rng.normal(0, 1.5, (7, 3))
    G = rng.normal(size=(7, mlp.P, mlp.C))
    g = mlp.backward(r, G)
    L = lambda m, rr: float(np.sum(m.forward(rr) * G))
    h = 1e-6
    for name, arr in (("grad_W1", mlp.W1), ("grad_W2", mlp.W2)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            lp = L(mlp, r)
            arr[idx] = old - h
            lm = L(mlp, r)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        assert np.abs(fd - g[name]).max() < 1e-7 * max(1, np.abs(fd).max()), name
    fd = np.zeros_like(r)
    for e in range(len(r)):
        for a in range(3):
            rp, rm = r.copy(), r.copy()
            rp[e, a] += h
            rm[e, a] -= h
            fd[e, a] = (L(mlp, rp) - L(mlp, rm)) / (2 * h)
    assert np.abs(fd - g["grad_r"]).max() < 1e-7 * max(1, np.abs(fd).max())
    # the radial part acts along r only: no component across it
    across = g["grad_r"] - np.sum(g["grad_r"] * r, axis=1, keepdims=True) * r / np.sum(r * r, axis=1, keepdims=True)
    assert np.abs(across).max() < 1e-12 * max(1, np.abs(g["grad_r"]).max())


def test_planted_mistake_is_caught():
    """Dropping the SiLU derivative changes grad_W1 beyond the central-difference tolerance."""
    mlp, rng = _mlp(2)
    r = rng.normal(0, 1.5, (5, 3))
    G = rng.normal(size=(5, mlp.P, mlp.C))
    good = mlp.backward(r, G)["grad_W1"]
    _, d, b, db, z = mlp._hidden(r)
    wrong = b.T @ (G.reshape(5, -1) @ mlp.W2.T)            # no SiLU' factor
    assert np.abs(wrong - good).max() > 1e-3


def test_whole_chain_forces_match_position_gradient():
    """E(pos) = sum out * G with out = TP(x, w(r), r) and w = MLP(|r|): the forces
    assembled from grad_r (through the harmonics) + grad_r (through the radial
    weights) equal minus the central differences of E in the positions."""
    rng = np.random.default_rng(7)
    n, e, L, C = 8, 30, 2, 3
    P = 15
    pos = rng.normal(0, 1.2, (n, 3))
    dst = rng.integers(0, n, e)
    src = (dst + rng.integers(1, n, e)) % n
    row_ptr, s, order = workloads.csr_from_pairs(n, dst, src)
    d = dst[order]
    mlp = radial.RadialMLP(rng.normal(size=(8, 6)) / np.sqrt(8), rng.normal(size=(6, P * C)) / np.sqrt(6), 4.0, P, C)
    x = rng.normal(size=(n, 9, C))
    G = rng.normal(size=(n, 9, C))
    tp = oracle.OracleTP("0..2", 2, "0..2", C)

    def energy(p):
        r = p[s] - p[d]
        return float(np.sum(tp.forward(row_ptr, s, r, x, mlp.forward(r)) * G))

    r = pos[s] - pos[d]
    w = mlp.forward(r)
    vjp = tp.backward(row_ptr, s, r, x, w, G, want=("w", "r"))
    g_total = vjp["grad_r"] + mlp.backward(r, vjp["grad_w"])["grad_r"]
    F, _ = oracle.assemble_forces(n, row_ptr, s, r, g_total)
    h = 1e-6
    fd = np.zeros_like(pos)
    for k in range(n):
        for a in range(3):
            pp, pm = pos.copy(), pos.copy()
            pp[k, a] += h
            pm[k, a] -= h
            fd[k, a] = -(energy(pp) - energy(pm)) / (2 * h)
    assert np.abs(F - fd).max() < 1e-7 * max(1, np.abs(fd).max())
    # the radial part matters: forces from the harmonics' part alone are off
    F_y, _ = oracle.assemble_forces(n, row_ptr, s, r, vjp["grad_r"])
    assert np.abs(F_y - fd).max() > 1e-3
