"""Pins of the oracle's second derivatives of the harmonics and of its VJP-of-VJP
(double backward), the second-order product that force-loss training needs
("FlashCart 如何让等变原子间势更快更准?", section "生成内核在高阶下胜过球谐基线").

The Hessian of Y(r/|r|) is pinned by central differences of the (already pinned)
gradient, by Euler's relation for a function of degree 0 (H r = -grad Y) and by the
angular Laplacian (trace H = -l(l+1) Y / |r|^2). The double backward is pinned by
central differences of <gg_x, grad_x> + <gg_w, grad_w> + <gg_r, grad_r> computed with
the oracle's first-order VJP, for each cotangent on its own, and by rotation
equivariance. Planted mistakes in the Hessian must fail the pins."""
import numpy as np
import pytest

import oracle
from oracle import cg, sh

LS = {2: [0, 1, 1, 1, 2, 2, 2, 2, 2], 3: [l for l in range(4) for _ in range(2 * l + 1)]}


def _rand_r(rng, n):
    return rng.standard_normal((n, 3)) * 1.7


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_sh_hess_matches_central_differences_of_the_gradient(lmax):
    rng = np.random.default_rng(lmax)
    r = _rand_r(rng, 7)
    H = sh.sh_hess(lmax, r)
    h = 1e-5
    fd = np.zeros_like(H)
    for b in range(3):
        d = np.zeros(3)
        d[b] = h
        fd[..., :, b] = (sh.sh_grad(lmax, r + d) - sh.sh_grad(lmax, r - d)) / (2 * h)
    assert np.max(np.abs(fd - H)) <= 1e-8 * max(1.0, np.max(np.abs(H)))
    assert np.max(np.abs(H - np.swapaxes(H, -1, -2))) < 1e-13


@pytest.mark.parametrize("lmax", [2, 3])
def test_sh_hess_euler_relation_and_laplacian(lmax):
    rng = np.random.default_rng(10 + lmax)
    r = _rand_r(rng, 9)
    H, G, Y = sh.sh_hess(lmax, r), sh.sh_grad(lmax, r), sh.sh(lmax, r)
    # Y(t r) = Y(r): d/dt of t (grad Y)(t r) . r at t = 1 gives H r + grad Y = 0
    assert np.max(np.abs(np.einsum("ekab,eb->eka", H, r) + G)) < 1e-12
    ls = np.asarray(LS[lmax] if lmax in LS else [], dtype=np.float64)
    lap = np.trace(H, axis1=-2, axis2=-1)
    assert np.max(np.abs(lap + ls * (ls + 1) * Y / np.sum(r * r, axis=1)[:, None])) < 1e-12


def test_sh_hess_zero_length_edge_is_zero():
    H = sh.sh_hess(3, np.zeros((2, 3)))
    assert np.all(H == 0.0)


@pytest.mark.parametrize("plant", ["dropped", "sign"])
def test_sh_hess_pins_catch_planted_mistakes(monkeypatch, plant):
    true = sh.sh_hess
    bad = (lambda l, r: 0.0 * true(l, r)) if plant == "dropped" else (lambda l, r: -true(l, r))
    monkeypatch.setattr(sh, "sh_hess", bad)
    r = _rand_r(np.random.default_rng(3), 5)
    H, G = sh.sh_hess(2, r), sh.sh_grad(2, r)
    assert np.max(np.abs(np.einsum("ekab,eb->eka", H, r) + G)) > 1e-3


def _problem(irreps, L, C, seed, n=6, deg=3, zero_edge=False):
    rng = np.random.default_rng(seed)
    tp = oracle.OracleTP(irreps, L, irreps, C)
    E = n * deg
    row_ptr = np.arange(0, E + 1, deg).astype(np.int32)
    src = rng.integers(0, n, E).astype(np.int32)
    r = _rand_r(rng, E)
    if zero_edge:
        r[1] = 0.0
    x = rng.standard_normal((n, tp.d_in, C))
    w = rng.standard_normal((E, tp.P, C))
    g = rng.standard_normal((n, tp.d_out, C))
    ct = {"gg_x": rng.standard_normal(x.shape), "gg_w": rng.standard_normal(w.shape),
          "gg_r": rng.standard_normal((E, 3))}
    return tp, rng, row_ptr, src, r, x, w, g, ct


def _phi(tp, row_ptr, src, r, x, w, g, ct):
    v = tp.backward(row_ptr, src, r, x, w, g)
    s = 0.0
    if ct.get("gg_x") is not None:
        s += np.sum(v["grad_x"] * ct["gg_x"])
    if ct.get("gg_w") is not None:
        s += np.sum(v["grad_w"] * ct["gg_w"])
    if ct.get("gg_r") is not None:
        s += np.sum(v["grad_r"] * ct["gg_r"])
    return s


def _check_fd(tp, rng, row_ptr, src, r, x, w, g, ct, frozen_edges=()):
    res = tp.double_backward(row_ptr, src, r, x, w, g, **ct)
    inputs = {"g": g, "x": x, "w": w, "r": r}
    for name, arr in inputs.items():
        d = rng.standard_normal(arr.shape)
        if name == "r":
            d[list(frozen_edges)] = 0.0      # no direction to differentiate at |r| = 0
        h = 1e-5 if name == "r" else 1.0     # linear in g, x, w: any step is exact
        plus = dict(inputs, **{name: arr + h * d})
        minus = dict(inputs, **{name: arr - h * d})
        fd = (_phi(tp, row_ptr, src, plus["r"], plus["x"], plus["w"], plus["g"], ct)
              - _phi(tp, row_ptr, src, minus["r"], minus["x"], minus["w"], minus["g"], ct)) / (2 * h)
        an = np.sum(res["grad_" + name] * d)
        tol = 1e-7 if name == "r" else 1e-11
        assert abs(fd - an) <= tol * max(1.0, abs(an)), (name, fd, an)
    return res


@pytest.mark.parametrize("which", ["gg_x", "gg_w", "gg_r", "all"])
@pytest.mark.parametrize("irreps,L,C", [("0..2", 2, 4), ("0e+1o+2e", 2, 3), ("0..3", 3, 2)])
def test_double_backward_matches_central_differences_of_the_vjp(which, irreps, L, C):
    tp, rng, row_ptr, src, r, x, w, g, ct = _problem(irreps, L, C, seed=len(irreps) * 7 + C)
    if which != "all":
        ct = {k: (v if k == which else None) for k, v in ct.items()}
    _check_fd(tp, rng, row_ptr, src, r, x, w, g, ct)


def test_double_backward_with_a_zero_length_edge():
    tp, rng, row_ptr, src, r, x, w, g, ct = _problem("0..2", 2, 4, seed=5, zero_edge=True)
    res = _check_fd(tp, rng, row_ptr, src, r, x, w, g, ct, frozen_edges=(1,))
    assert np.all(res["grad_r"][1] == 0.0)   # no gradient through a direction that does not exist


def test_double_backward_is_rotation_equivariant():
    tp, rng, row_ptr, src, r, x, w, g, ct = _problem("0..2", 2, 3, seed=11)
    R = cg.random_rotation(rng)
    D = np.zeros((tp.d_in, tp.d_in))
    for l in range(3):
        D[l * l:(l + 1) * (l + 1), l * l:(l + 1) * (l + 1)] = cg.wigner_d(l, R)
    rot = lambda a: np.einsum("ab,nbc->nac", D, a)
    a = tp.double_backward(row_ptr, src, r, x, w, g, **ct)
    b = tp.double_backward(row_ptr, src, r @ R.T, rot(x), w, rot(g), gg_x=rot(ct["gg_x"]), gg_w=ct["gg_w"],
                           gg_r=ct["gg_r"] @ R.T)
    scale = max(np.max(np.abs(a[k])) for k in a)
    assert np.max(np.abs(b["grad_g"] - rot(a["grad_g"]))) < 1e-10 * scale
    assert np.max(np.abs(b["grad_x"] - rot(a["grad_x"]))) < 1e-10 * scale
    assert np.max(np.abs(b["grad_w"] - a["grad_w"])) < 1e-10 * scale
    assert np.max(np.abs(b["grad_r"] - a["grad_r"] @ R.T)) < 1e-10 * scale


def test_double_backward_pin_catches_a_dropped_hessian_term(monkeypatch):
    tp, rng, row_ptr, src, r, x, w, g, ct = _problem("0..2", 2, 4, seed=2)
    ct = {"gg_x": None, "gg_w": None, "gg_r": ct["gg_r"]}
    true = sh.sh_hess
    monkeypatch.setattr(sh, "sh_hess", lambda l, rr: 0.0 * true(l, rr))
    with pytest.raises(AssertionError):
        _check_fd(tp, rng, row_ptr, src, r, x, w, g, ct)
