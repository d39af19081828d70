"""Pins of the oracle's real coupling tensors (oracle/cg.py) and path list (oracle/paths.py)."""
import itertools

import numpy as np
import pytest

from oracle import cg, paths, sh

LMAX = 3
TRIPLES = [(a, b, c) for a, b, c in itertools.product(range(LMAX + 1), repeat=3) if cg.triangle(a, b, c)]


def test_closed_forms_up_to_l1():
    assert np.allclose(cg.real_cg(0, 0, 0), np.ones((1, 1, 1)))
    for l in range(0, LMAX + 1):
        d = 2 * l + 1
        assert np.allclose(cg.real_cg(0, l, l)[0], np.eye(d), atol=1e-13)
        assert np.allclose(cg.real_cg(l, 0, l)[:, 0, :], np.eye(d), atol=1e-13)
    assert np.allclose(cg.real_cg(1, 1, 0)[:, :, 0], np.eye(3) / np.sqrt(3), atol=1e-13)
    eps = np.zeros((3, 3, 3))
    for (a, b, c), s in {(0, 1, 2): 1, (1, 2, 0): 1, (2, 0, 1): 1,
                         (0, 2, 1): -1, (2, 1, 0): -1, (1, 0, 2): -1}.items():
        eps[a, b, c] = s
    assert np.allclose(cg.real_cg(1, 1, 1), eps / np.sqrt(2), atol=1e-13)


@pytest.mark.parametrize("l1,l2", list(itertools.product(range(LMAX + 1), repeat=2)))
def test_orthogonality_and_completeness(l1, l2):
    """sum_{m1 m2} C^{l3} C^{l3'} = delta delta, and the l3 blocks span x (x) y."""
    blocks = [cg.real_cg(l1, l2, l3).reshape((2 * l1 + 1) * (2 * l2 + 1), -1)
              for l3 in range(abs(l1 - l2), l1 + l2 + 1)]
    M = np.concatenate(blocks, axis=1)           # [(d1 d2), sum d3], square
    assert M.shape[0] == M.shape[1]
    assert np.allclose(M.T @ M, np.eye(M.shape[1]), atol=1e-12)
    assert np.allclose(M @ M.T, np.eye(M.shape[0]), atol=1e-12)


def test_off_triangle_is_zero():
    for a, b, c in itertools.product(range(LMAX + 1), repeat=3):
        if not cg.triangle(a, b, c):
            assert not np.any(cg.real_cg(a, b, c))


@pytest.mark.parametrize("l1,l2,l3", TRIPLES)
def test_sign_rule_and_azimuthal_selection(l1, l2, l3):
    c = cg.real_cg(l1, l2, l3)
    assert c.reshape(-1)[np.flatnonzero(c)[0]] > 0
    for m1, m2, m3 in np.argwhere(c != 0):
        a, b, o = abs(m1 - l1), abs(m2 - l2), abs(m3 - l3)
        assert o in (abs(a - b), a + b), (m1, m2, m3)


@pytest.mark.parametrize("l1,l2,l3", [t for t in TRIPLES if sum(t) % 2 == 0])
def test_gaunt_product_identity(l1, l2, l3):
    """For even l1+l2+l3: sum CG Y_l1(u) Y_l2(u) is a constant multiple of Y_l3(u)."""
    r = np.random.default_rng(5).standard_normal((40, 3))
    lhs = np.einsum("abc,na,nb->nc", cg.real_cg(l1, l2, l3), sh.sh_block(l1, r), sh.sh_block(l2, r))
    rhs = sh.sh_block(l3, r)
    k = np.sum(lhs * rhs) / np.sum(rhs * rhs)
    assert abs(k) > 1e-3
    assert np.allclose(lhs, k * rhs, atol=1e-11)


@pytest.mark.parametrize("l1,l2,l3", TRIPLES)
def test_equivariance_fresh_rotations(l1, l2, l3):
    """CG(D1 x, D2 y) = D3 CG(x, y) for rotations and directions the construction never saw."""
    rng = np.random.default_rng(777 + l1 * 16 + l2 * 4 + l3)
    R = cg.random_rotation(rng)
    c = cg.real_cg(l1, l2, l3)
    D1, D2, D3 = (cg.wigner_d(l, R, seed=999) for l in (l1, l2, l3))
    x, y = rng.standard_normal(2 * l1 + 1), rng.standard_normal(2 * l2 + 1)
    lhs = np.einsum("abc,a,b->c", c, D1 @ x, D2 @ y)
    rhs = D3 @ np.einsum("abc,a,b->c", c, x, y)
    assert np.allclose(lhs, rhs, atol=1e-12)


def test_wigner_d_l1_is_the_rotation_in_yzx_order():
    R = cg.random_rotation(np.random.default_rng(3))
    perm = [1, 2, 0]
    assert np.allclose(cg.wigner_d(1, R), R[np.ix_(perm, perm)], atol=1e-13)


def test_path_counts_and_order():
    for L, P in [(0, 1), (1, 5), (2, 15), (3, 34)]:
        ps = paths.enumerate_paths(f"0..{L}", L, f"0..{L}")
        assert len(ps) == P and ps == sorted(ps)
    assert paths.enumerate_paths("0+1", 1, "0+1") == [(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 0), (1, 1, 1)]
    o3 = paths.enumerate_paths("0e+1o+2e+3o", 3, "0e+1o+2e+3o")
    assert all(sum(p) % 2 == 0 for p in o3) and len(o3) == 23
    assert [len(paths.enumerate_paths(f"0e+1o+2e+3o"[:k], l, f"0e+1o+2e+3o"[:k]))
            for k, l in [(2, 0), (5, 1), (8, 2)]] == [1, 4, 11]


def test_nnz_totals():
    tot = {L: sum(len(cg.nnz_list(*p)) for p in paths.enumerate_paths(f"0..{L}", L, f"0..{L}"))
           for L in (1, 2, 3)}
    # selection-rule upper bounds are 17 / 141 / 652; the exact counts are below them
    assert tot[1] <= 17 and tot[2] <= 141 and tot[3] <= 652
    assert tot == {1: 16, 2: 137, 3: 611}
