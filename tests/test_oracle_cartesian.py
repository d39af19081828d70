"""Pins of the Cartesian form of the edge-wise tensor product ("FlashCart
如何让等变原子间势更快更准?", sections "FlashCart 用笛卡尔内核替代球谐耦合" and
"生成内核在高阶下胜过球谐基线"): the STF projector against its closed forms, the
Cartesian edge attribute against the (pinned) spherical harmonics, every path's coupling
against the spherical Clebsch-Gordan coupling up to one constant (Schur), closed forms of
the low-rank paths, rotation equivariance in Cartesian form, the whole edge convolution
against the spherical oracle with per-path rescaled weights, and the VJP against central
differences. A planted mistake (no STF projection) must fail."""
import numpy as np
import pytest
import torch

import oracle
from oracle import cartesian as ct
from oracle import cg, sh

D64 = torch.float64


def _stf_rand(rng, lead, l):
    A = torch.from_numpy(rng.standard_normal(tuple(lead) + (3,) * l))
    return ct.stf(A, l)


def _sph(A, l):
    return ct.to_spherical(A, l) if l > 0 else A.reshape(*A.shape, 1)


def test_stf_projector_closed_forms():
    rng = np.random.default_rng(0)
    for l in range(5):
        P = ct.stf_projector(l)
        assert np.allclose(P @ P, P, atol=1e-13) and np.allclose(P, P.T, atol=1e-13)
        assert round(np.trace(P)) == 2 * l + 1
    T = torch.from_numpy(rng.standard_normal((3, 3)))
    S = (T + T.T) / 2
    assert torch.allclose(ct.stf(T, 2), S - torch.eye(3, dtype=D64) * torch.trace(S) / 3, atol=1e-14)
    T3 = torch.from_numpy(rng.standard_normal((3, 3, 3)))
    S3 = sum(T3.permute(*p) for p in [(0, 1, 2), (0, 2, 1), (1, 0, 2), (1, 2, 0), (2, 0, 1), (2, 1, 0)]) / 6
    v = torch.einsum("aab->b", S3)
    d = torch.eye(3, dtype=D64)
    ref = S3 - (torch.einsum("ab,c->abc", d, v) + torch.einsum("ac,b->abc", d, v) + torch.einsum("bc,a->abc", d, v)) / 5
    assert torch.allclose(ct.stf(T3, 3), ref, atol=1e-14)


@pytest.mark.parametrize("l", [0, 1, 2, 3])
def test_edge_attribute_is_the_spherical_harmonic_in_cartesian_components(l):
    r = np.random.default_rng(l).standard_normal((11, 3)) * 1.3
    r[2] = 0.0
    got = _sph(ct.edge_attr(torch.from_numpy(r), l), l)
    assert np.max(np.abs(got.numpy() - sh.sh_block(l, r))) < 1e-14


def _all_paths(L):
    return oracle.OracleTP(f"0..{L}", L, f"0..{L}", 1).paths


@pytest.mark.parametrize("path", _all_paths(3))
def test_every_path_is_the_clebsch_gordan_coupling_up_to_one_constant(path):
    l1, l2, l3 = path
    rng = np.random.default_rng(l1 * 100 + l2 * 10 + l3)
    A = _stf_rand(rng, (25,), l1)
    r = torch.from_numpy(rng.standard_normal((25, 3)))
    B = ct.edge_attr(r, l2).reshape(25, *([3] * l2))
    cart = _sph(ct.couple(A, B, l1, l2, l3), l3)
    sphr = torch.einsum("abc,na,nb->nc", torch.from_numpy(cg.real_cg(l1, l2, l3)), _sph(A, l1),
                        torch.from_numpy(sh.sh_block(l2, r.numpy())))
    c = float((cart * sphr).sum() / (sphr * sphr).sum())
    assert abs(c) > 1e-3                                   # the coupling is not identically zero
    assert float((cart - c * sphr).abs().max()) < 1e-12 * float(cart.abs().max())


def _assert_stf(T, l):
    """Symmetric under every index swap and traceless over every index pair (l >= 2)."""
    lead = T.dim() - l
    scale = max(1.0, float(T.abs().max()))
    for i in range(l):
        for j in range(i + 1, l):
            assert float((T - T.transpose(lead + i, lead + j)).abs().max()) < 1e-12 * scale
            assert float(torch.diagonal(T, dim1=lead + i, dim2=lead + j).sum(-1).abs().max()) < 1e-12 * scale


@pytest.mark.parametrize("path", [p for p in _all_paths(3) if p[2] >= 2])
def test_every_path_output_is_symmetric_traceless(path):
    l1, l2, l3 = path
    rng = np.random.default_rng(l1 * 100 + l2 * 10 + l3 + 1)
    A = _stf_rand(rng, (9,), l1)
    B = ct.edge_attr(torch.from_numpy(rng.standard_normal((9, 3))), l2).reshape(9, *([3] * l2))
    _assert_stf(ct.couple(A, B, l1, l2, l3), l3)


def test_low_rank_paths_closed_forms():
    rng = np.random.default_rng(7)
    a = torch.from_numpy(rng.standard_normal((6, 3)))
    s = torch.from_numpy(rng.standard_normal(6))
    r = torch.from_numpy(rng.standard_normal((6, 3)))
    u = r / torch.linalg.norm(r, dim=1, keepdim=True)
    Au = _stf_rand(rng, (6,), 2)
    assert torch.allclose(ct.couple(a, u, 1, 1, 0), (a * u).sum(1), atol=1e-14)
    assert torch.allclose(ct.couple(a, u, 1, 1, 1), torch.linalg.cross(a, u), atol=1e-14)
    assert torch.allclose(ct.couple(a, torch.ones(6, dtype=D64), 1, 0, 1), a, atol=1e-14)
    assert torch.allclose(ct.couple(s, u, 0, 1, 1), s[:, None] * u, atol=1e-14)
    sym = (a[:, :, None] * u[:, None, :] + a[:, None, :] * u[:, :, None]) / 2
    ref = sym - torch.eye(3, dtype=D64) * (a * u).sum(1)[:, None, None] / 3
    assert torch.allclose(ct.couple(a, u, 1, 1, 2), ref, atol=1e-14)
    assert torch.allclose(ct.couple(Au, u, 2, 1, 1), torch.einsum("nab,nb->na", Au, u), atol=1e-14)


def _graph(rng, n=7, deg=3):
    E = n * deg
    row_ptr = np.arange(0, E + 1, deg)
    src = rng.integers(0, n, E)
    return n, E, row_ptr, src


def _rot(T, R, l):
    for i in range(l):  # rotate every tensor index
        T = torch.movedim(torch.tensordot(T, R.T, dims=([T.dim() - l + i], [0])), -1, T.dim() - l + i)
    return T


def test_edge_convolution_is_rotation_equivariant():
    rng = np.random.default_rng(3)
    tp = ct.OracleCartTP("0..2", 2, "0..2", 3)
    n, E, row_ptr, src = _graph(rng)
    r = torch.from_numpy(rng.standard_normal((E, 3)))
    x = {l: _stf_rand(rng, (n, 3), l) for l in range(3)}
    w = torch.from_numpy(rng.standard_normal((E, tp.P, 3)))
    R = torch.from_numpy(cg.random_rotation(rng))
    a = tp.forward(row_ptr, src, r, x, w)
    b = tp.forward(row_ptr, src, r @ R.T, {l: _rot(v, R, l) for l, v in x.items()}, w)
    for l in a:
        assert torch.allclose(b[l], _rot(a[l], R, l), atol=1e-12)


@pytest.mark.parametrize("irreps,L", [("0..2", 2), ("0..3", 3), ("0e+1o+2e", 2)])
def test_edge_convolution_equals_the_spherical_one_with_rescaled_weights(irreps, L):
    rng = np.random.default_rng(L)
    C = 2
    tp_c = ct.OracleCartTP(irreps, L, irreps, C)
    tp_s = oracle.OracleTP(irreps, L, irreps, C)
    assert tp_c.paths == tp_s.paths
    n, E, row_ptr, src = _graph(rng)
    r = rng.standard_normal((E, 3))
    x = {l: _stf_rand(rng, (n, C), l) for l in tp_c.ls_in}
    w = rng.standard_normal((E, tp_c.P, C))
    # one constant per path, from one probe of that path alone
    scale = []
    for l1, l2, l3 in tp_c.paths:
        A = _stf_rand(rng, (4,), l1)
        rr = torch.from_numpy(rng.standard_normal((4, 3)))
        cart = _sph(ct.couple(A, ct.edge_attr(rr, l2).reshape(4, *([3] * l2)), l1, l2, l3), l3)
        sphr = torch.einsum("abc,na,nb->nc", torch.from_numpy(cg.real_cg(l1, l2, l3)), _sph(A, l1),
                            torch.from_numpy(sh.sh_block(l2, rr.numpy())))
        scale.append(float((cart * sphr).sum() / (sphr * sphr).sum()))
    out_c = tp_c.forward(row_ptr, src, r, x, w)
    x_s = np.concatenate([_sph(x[l], l).permute(0, 2, 1).numpy() for l in tp_c.ls_in], axis=1)
    out_s = tp_s.forward(row_ptr.astype(np.int32), src.astype(np.int32), r, x_s,
                         w * np.asarray(scale)[None, :, None])
    got = np.concatenate([_sph(out_c[l], l).permute(0, 2, 1).numpy() for l in tp_c.ls_out], axis=1)
    assert np.max(np.abs(got - out_s)) < 1e-12 * np.max(np.abs(out_s))


def test_vjp_matches_central_differences():
    rng = np.random.default_rng(9)
    tp = ct.OracleCartTP("0..2", 2, "0..2", 2)
    n, E, row_ptr, src = _graph(rng, n=5)
    r = torch.from_numpy(rng.standard_normal((E, 3)))
    x = {l: _stf_rand(rng, (n, 2), l) for l in range(3)}
    w = torch.from_numpy(rng.standard_normal((E, tp.P, 2)))
    g = {l: _stf_rand(rng, (n, 2), l) for l in range(3)}
    res = tp.backward(row_ptr, src, r, x, w, g)

    def L(x_, w_, r_):
        out = tp.forward(row_ptr, src, r_, x_, w_)
        return float(sum((out[l] * g[l]).sum() for l in out))

    dx = {l: _stf_rand(rng, (n, 2), l) for l in range(3)}
    fd = (L({l: x[l] + dx[l] for l in x}, w, r) - L({l: x[l] - dx[l] for l in x}, w, r)) / 2
    an = float(sum((res["grad_x"][l] * dx[l]).sum() for l in x))
    assert abs(fd - an) < 1e-11 * max(1.0, abs(an))
    dw = torch.from_numpy(rng.standard_normal(w.shape))
    fd = (L(x, w + dw, r) - L(x, w - dw, r)) / 2
    assert abs(fd - float((res["grad_w"] * dw).sum())) < 1e-11 * max(1.0, abs(fd))
    dr = torch.from_numpy(rng.standard_normal(r.shape))
    h = 1e-6
    fd = (L(x, w, r + h * dr) - L(x, w, r - h * dr)) / (2 * h)
    assert abs(fd - float((res["grad_r"] * dr).sum())) < 1e-7 * max(1.0, abs(fd))


def test_pin_catches_a_missing_stf_projection(monkeypatch):
    # the spherical components cannot see it (an STF tensor contracted with any tensor
    # sees only its STF part); the Cartesian output check does
    monkeypatch.setattr(ct, "stf", lambda T, l: T)
    test_every_path_is_the_clebsch_gordan_coupling_up_to_one_constant((1, 1, 2))
    with pytest.raises(AssertionError):
        test_every_path_output_is_symmetric_traceless((1, 1, 2))
