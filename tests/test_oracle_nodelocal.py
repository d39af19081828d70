"""Pins of the node-local product oracle (oracle/nodelocal.py; "FlashCart
如何让等变原子间势更快更准?", sections "FlashCart 用笛卡尔内核替代球谐耦合" and
"生成内核在高阶下胜过球谐基线"): order 1 is the identity; the scalar product has the closed
form x^K times the product of the step weights; two-step ladders of rank-1 features have
closed forms in both forms (dot product, then scaling; the STF square of a vector, then its
contraction with the vector; a cross product through the Levi-Civita symbol), taken in
both step orders so that a ladder that reads its weights in the wrong order fails; the
Cartesian product equals the spherical one once each path's weight is rescaled by the
constant that relates the two couplings (Schur); both forms are rotation equivariant.
Planted mistakes (a ladder that multiplies by its own last step instead of by x, one that
reads its steps' weights backwards) must fail."""
import numpy as np
import pytest
import torch

from oracle import cartesian as ct
from oracle import cg
from oracle import nodelocal as nl

D64 = torch.float64
YZX = [1, 2, 0]          # real spherical order of rank 1: (y, z, x)


def _stf_rand(rng, lead, l):
    return ct.stf(torch.from_numpy(rng.standard_normal(tuple(lead) + (3,) * l)), l)


def _sph(A, l):
    return ct.to_spherical(A, l) if l > 0 else A.reshape(*A.shape, 1)


def _weights(paths, K, C, only=None):
    """w [K-1, P, C]; with ``only`` = {step: {path: [C] values}} every other weight is 0."""
    w = np.zeros((K - 1, len(paths), C))
    for k, d in (only or {}).items():
        for p, v in d.items():
            w[k, paths.index(p)] = v
    return w


def test_paths_follow_the_triangle_and_parity_rules():
    assert len(nl.node_paths("0..3")) == 34
    assert nl.node_paths("0..1") == [(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 0), (1, 1, 1)]
    assert nl.node_paths("0e+1o") == [(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 0)]
    assert all((a + b + c) % 2 == 0 for a, b, c in nl.node_paths("0e+1o+2e+3o"))


@pytest.mark.parametrize("irreps", ["0..3", "0e+1o+2e"])
def test_order_one_is_the_identity(irreps):
    rng = np.random.default_rng(0)
    D = sum(2 * l + 1 for l in nl._ranks(irreps))
    x = rng.standard_normal((5, D, 3))
    assert np.array_equal(nl.node_product(x, np.zeros((0, len(nl.node_paths(irreps)), 3)), irreps), x)
    xc = {l: _stf_rand(rng, (5, 3), l) for l in nl._ranks(irreps)}
    out = nl.node_product_cartesian(xc, np.zeros((0, len(nl.node_paths(irreps)), 3)), irreps)
    for l in xc:
        assert torch.equal(out[l], xc[l])


@pytest.mark.parametrize("K", [2, 3, 5])
def test_scalar_closed_form(K):
    rng = np.random.default_rng(K)
    x = rng.standard_normal((7, 1, 4))
    w = rng.standard_normal((K - 1, 1, 4))
    want = x[:, 0, :] ** K * np.prod(w[:, 0, :], axis=0)[None, :]
    assert np.allclose(nl.node_product(x, w, "0")[:, 0, :], want, rtol=1e-13, atol=0)
    got = nl.node_product_cartesian({0: torch.from_numpy(x[:, 0, :])}, w, "0")[0].numpy()
    assert np.allclose(got, want, rtol=1e-13, atol=0)


def _vec_input(rng, N, C):
    s = rng.standard_normal((N, C))
    v = rng.standard_normal((N, C, 3))
    x = np.zeros((N, 4, C))
    x[:, 0, :] = s
    x[:, 1:4, :] = np.moveaxis(v[..., YZX], 2, 1)
    return s, v, x


def test_spherical_two_step_ladder_closed_forms():
    """Rank 0 and 1 in an orthonormal real basis: the (1,1,0) coupling is the dot product
    over sqrt(3) and the (0,1,1) coupling is the scaling (unit normalisation over m1, m2,
    first nonzero coefficient positive)."""
    rng = np.random.default_rng(1)
    N, C = 6, 3
    s, v, x = _vec_input(rng, N, C)
    a, b = rng.standard_normal(C), rng.standard_normal(C)
    paths = nl.node_paths("0..1")
    vv = (v * v).sum(-1)
    # dot first, then scale: B3_1 = a b |v|^2 v / sqrt(3), B3_0 = 0
    out = nl.node_product(x, _weights(paths, 3, C, {0: {(1, 1, 0): a}, 1: {(0, 1, 1): b}}), "0..1")
    want1 = (a * b)[None, :, None] * vv[..., None] * v / np.sqrt(3)
    assert np.allclose(out[:, 1:4, :], np.moveaxis(want1[..., YZX], 2, 1), rtol=0, atol=1e-13)
    assert np.max(np.abs(out[:, 0, :])) == 0.0
    # scale first, then dot: B3_0 = a b s |v|^2 / sqrt(3), B3_1 = 0
    out = nl.node_product(x, _weights(paths, 3, C, {0: {(0, 1, 1): b}, 1: {(1, 1, 0): a}}), "0..1")
    assert np.allclose(out[:, 0, :], (a * b)[None, :] * s * vv / np.sqrt(3), rtol=0, atol=1e-13)
    assert np.max(np.abs(out[:, 1:4, :])) == 0.0


def test_cartesian_two_step_ladder_closed_forms():
    rng = np.random.default_rng(2)
    N, C = 6, 3
    v = torch.from_numpy(rng.standard_normal((N, C, 3)))
    M = _stf_rand(rng, (N, C), 2)
    s = torch.from_numpy(rng.standard_normal((N, C)))
    x = {0: s, 1: v, 2: M}
    a, b = rng.standard_normal(C), rng.standard_normal(C)
    ab = torch.from_numpy(a * b)[None, :, None]
    paths = nl.node_paths("0..2")
    vv = (v * v).sum(-1, keepdim=True)
    # STF square of v, then contracted with v: (v v^T - |v|^2 I / 3) v = 2/3 |v|^2 v
    out = nl.node_product_cartesian(x, _weights(paths, 3, C, {0: {(1, 1, 2): a}, 1: {(2, 1, 1): b}}), "0..2")
    assert torch.allclose(out[1], ab * (2.0 / 3.0) * vv * v, rtol=0, atol=1e-13)
    assert float(out[0].abs().max()) == 0.0 and float(out[2].abs().max()) == 0.0
    # v crossed (through epsilon) with the columns of M, then the STF part: path (1, 2, 2)
    out = nl.node_product_cartesian(x, _weights(paths, 2, C, {0: {(1, 2, 2): a}}), "0..2")
    Q = torch.linalg.cross(v[:, :, :, None].expand(-1, -1, -1, 3), M, dim=2)      # Q[.., n, b] = (v x M[:, b])_n
    Q = Q.transpose(2, 3)                                                       # [.., b, n]
    S = (Q + Q.transpose(2, 3)) / 2
    want = S - torch.eye(3, dtype=D64) * torch.einsum("ncaa->nc", S)[..., None, None] / 3
    assert torch.allclose(out[2], torch.from_numpy(a)[None, :, None, None] * want, rtol=0, atol=1e-13)
    # scaled by s first, then dotted with v: the other step order
    out = nl.node_product_cartesian(x, _weights(paths, 3, C, {0: {(0, 1, 1): b}, 1: {(1, 1, 0): a}}), "0..2")
    assert torch.allclose(out[0], ab[..., 0] * s * vv[..., 0], rtol=0, atol=1e-13)


def _path_scale(rng, l1, l2, l3):
    """The constant c with to_spherical(couple(A, B)) = c * CG(to_spherical(A), to_spherical(B))."""
    A, B = _stf_rand(rng, (4,), l1), _stf_rand(rng, (4,), l2)
    cart = _sph(ct.couple(A, B, l1, l2, l3), l3)
    sphr = torch.einsum("abc,na,nb->nc", torch.from_numpy(cg.real_cg(l1, l2, l3)), _sph(A, l1), _sph(B, l2))
    c = float((cart * sphr).sum() / (sphr * sphr).sum())
    assert float((cart - c * sphr).abs().max()) < 1e-12 * float(cart.abs().max())
    return c


@pytest.mark.parametrize("irreps,K", [("0..2", 4), ("0..3", 3), ("0e+1o+2e+3o", 4)])
def test_cartesian_equals_spherical_with_rescaled_weights(irreps, K):
    rng = np.random.default_rng(K + len(irreps))
    C, N = 3, 5
    paths = nl.node_paths(irreps)
    ls = nl._ranks(irreps)
    scale = np.array([_path_scale(rng, *p) for p in paths])
    x = {l: _stf_rand(rng, (N, C), l) for l in ls}
    w = rng.standard_normal((K - 1, len(paths), C)) / np.sqrt(len(paths))
    out_c = nl.node_product_cartesian(x, w, irreps)
    x_s = np.concatenate([_sph(x[l], l).permute(0, 2, 1).numpy() for l in ls], axis=1)
    out_s = nl.node_product(x_s, w * scale[None, :, None], irreps)
    got = np.concatenate([_sph(out_c[l], l).permute(0, 2, 1).numpy() for l in ls], axis=1)
    assert np.max(np.abs(got - out_s)) < 1e-12 * np.max(np.abs(out_s))


def _rot(T, R, l):
    for i in range(l):
        T = torch.movedim(torch.tensordot(T, R.T, dims=([T.dim() - l + i], [0])), -1, T.dim() - l + i)
    return T


def test_both_forms_are_rotation_equivariant():
    rng = np.random.default_rng(5)
    irreps, K, C, N = "0..3", 4, 2, 4
    paths = nl.node_paths(irreps)
    w = rng.standard_normal((K - 1, len(paths), C))
    R = cg.random_rotation(rng)
    x = rng.standard_normal((N, 16, C))
    Dm = np.zeros((16, 16))
    for l in range(4):
        Dm[l * l:(l + 1) ** 2, l * l:(l + 1) ** 2] = cg.wigner_d(l, R, seed=77)
    a = nl.node_product(x, w, irreps)
    b = nl.node_product(np.einsum("ij,njc->nic", Dm, x), w, irreps)
    assert np.allclose(b, np.einsum("ij,njc->nic", Dm, a), atol=1e-11 * np.max(np.abs(a)))
    Rt = torch.from_numpy(R)
    xc = {l: _stf_rand(rng, (N, C), l) for l in range(4)}
    ac = nl.node_product_cartesian(xc, w, irreps)
    bc = nl.node_product_cartesian({l: _rot(t, Rt, l) for l, t in xc.items()}, w, irreps)
    for l in ac:
        assert torch.allclose(bc[l], _rot(ac[l], Rt, l), atol=1e-11 * float(ac[l].abs().max()))


def test_pins_catch_a_ladder_on_its_own_output(monkeypatch):
    sph, cart = nl._spherical_step, nl._cartesian_step
    monkeypatch.setattr(nl, "_spherical_step", lambda B, X, wk, paths: sph(B, B, wk, paths))
    monkeypatch.setattr(nl, "_cartesian_step", lambda B, X, wk, paths, C: cart(B, B, wk, paths, C))
    with pytest.raises(AssertionError):
        test_scalar_closed_form(3)
    with pytest.raises(AssertionError):
        test_spherical_two_step_ladder_closed_forms()
    with pytest.raises(AssertionError):
        test_cartesian_two_step_ladder_closed_forms()


def test_pins_catch_weights_read_backwards(monkeypatch):
    prod, prod_c = nl.node_product, nl.node_product_cartesian
    monkeypatch.setattr(nl, "node_product", lambda x, w, irreps: prod(x, np.asarray(w)[::-1].copy(), irreps))
    monkeypatch.setattr(nl, "node_product_cartesian", lambda x, w, irreps: prod_c(x, np.asarray(w)[::-1].copy(), irreps))
    with pytest.raises(AssertionError):
        test_spherical_two_step_ladder_closed_forms()
    with pytest.raises(AssertionError):
        test_cartesian_two_step_ladder_closed_forms()
