"""FP64 oracle for the Cartesian form of the edge-wise tensor product.
TEST INFRASTRUCTURE ONLY (same rule as the rest of oracle/).

FlashCart writes the equivariant tensor product in independent Cartesian
components instead of spherical-harmonic couplings, and compares its edge
convolution with spherical implementations at equal tensor rank
("FlashCart 如何让等变原子间势更快更准?", sections "FlashCart 用笛卡尔内核替代球谐耦合"
and "生成内核在高阶下胜过球谐基线"). The pages give no formulas. The plain reading taken
here, one irreducible Cartesian tensor per rank:

  * a feature of rank l is a symmetric traceless (STF) tensor with l indices of size
    3, held as a full 3^l array (2l+1 independent components);
  * the edge attribute of rank l is the STF part of u (x) ... (x) u (l factors), u = r/|r|
    (rank 0: 1; an edge shorter than 1e-12 gives 0 for l >= 1);
  * the path (l1, l2 -> l3) contracts k index pairs of the two operands, with
    k = (l1 + l2 - l3) / 2 for l1 + l2 + l3 even; for l1 + l2 + l3 odd it contracts
    k = (l1 + l2 - l3 - 1) / 2 pairs and one more pair through the Levi-Civita symbol,
    whose third index is a new output index; the STF part of the l3 remaining indices
    is the path's output. No normalisation constant;
  * the edge convolution is the spherical one with these couplings:
        out[i][l3][c] = sum_{e: i <- j} sum_{p = (l1, l2, l3)} w[e, p, c] coupling_p(x[j][l1][c], Y_l2(e)).

By Schur's lemma each path's Cartesian coupling equals the spherical Clebsch-Gordan
coupling up to one constant per path, once both are written in the same components
(``to_spherical`` below); the tests pin exactly that, rotation equivariance in Cartesian
form, and closed forms of the low-rank paths. The VJP is reverse-mode automatic
differentiation (torch.autograd in float64) of this forward.
"""
from __future__ import annotations

import itertools
import string
from functools import lru_cache
from math import factorial

import numpy as np
import torch

from . import paths as paths_mod
from . import sh as sh_mod

R_EPS = 1e-12


@lru_cache(maxsize=None)
def stf_projector(l: int) -> np.ndarray:
    """Orthogonal projector [3^l, 3^l] onto the symmetric traceless tensors of rank l.

    The subspace is the symmetric tensors whose every trace over an index pair is zero:
    the null space, within the range of the symmetriser, of the trace maps.
    """
    n = 3 ** l
    if l < 2:
        return np.eye(n)
    idx = list(itertools.product(range(3), repeat=l))
    pos = {t: i for i, t in enumerate(idx)}
    sym = np.zeros((n, n))
    perms = list(itertools.permutations(range(l)))
    for t in idx:
        for p in perms:
            sym[pos[t], pos[tuple(t[q] for q in p)]] += 1.0 / len(perms)
    # trace over the first two indices (enough for symmetric tensors): [3^(l-2), 3^l]
    tr = np.zeros((3 ** (l - 2), n))
    rest = list(itertools.product(range(3), repeat=l - 2))
    for i, t in enumerate(rest):
        for a in range(3):
            tr[i, pos[(a, a) + t]] = 1.0
    # basis of symmetric tensors, then the part of it that the trace annihilates
    u, s, _ = np.linalg.svd(sym)
    B = u[:, s > 0.5]                       # orthonormal basis of the symmetric subspace
    _, s2, vt = np.linalg.svd(tr @ B)
    rank = int(np.sum(s2 > 1e-10))
    N = vt[rank:].T                         # coordinates (in B) of the traceless ones
    Q = B @ N                               # orthonormal basis of STF, [3^l, 2l+1]
    assert Q.shape[1] == 2 * l + 1
    return Q @ Q.T


def stf(T: torch.Tensor, l: int) -> torch.Tensor:
    """STF part of the trailing l indices of T."""
    if l < 2:
        return T
    lead = T.shape[: T.dim() - l]
    P = torch.from_numpy(stf_projector(l)).to(T.dtype)
    return (T.reshape(*lead, 3 ** l) @ P.T).reshape(*lead, *([3] * l))


def levi_civita(dtype=torch.float64) -> torch.Tensor:
    e = torch.zeros(3, 3, 3, dtype=dtype)
    for (a, b, c), s in (((0, 1, 2), 1), ((1, 2, 0), 1), ((2, 0, 1), 1), ((0, 2, 1), -1), ((2, 1, 0), -1),
                         ((1, 0, 2), -1)):
        e[a, b, c] = s
    return e


def couple(A: torch.Tensor, B: torch.Tensor, l1: int, l2: int, l3: int) -> torch.Tensor:
    """Path (l1, l2 -> l3) of two batches of STF tensors (trailing l1 / l2 indices, same
    leading shape): k contractions (+ one through epsilon when l1 + l2 + l3 is odd), STF."""
    odd = (l1 + l2 + l3) % 2
    k = (l1 + l2 - l3 - odd) // 2
    assert k >= 0 and l1 - k - odd >= 0 and l2 - k - odd >= 0, (l1, l2, l3)
    letters = iter(string.ascii_lowercase[1:])
    a_idx = [next(letters) for _ in range(l1)]
    b_idx = a_idx[l1 - k:] + [next(letters) for _ in range(l2 - k)]   # first k of B = last k of A
    free_a = a_idx[: l1 - k]
    free_b = b_idx[k:]
    lead = "Z"
    if odd:
        ea, eb, new = free_a[-1], free_b[0], next(letters)
        out = free_a[:-1] + free_b[1:] + [new]
        spec = f"{lead}{''.join(a_idx)},{lead}{''.join(b_idx)},{ea}{eb}{new}->{lead}{''.join(out)}"
        lead_shape = A.shape[: A.dim() - l1]
        res = torch.einsum(spec, A.reshape(-1, *A.shape[A.dim() - l1:]), B.reshape(-1, *B.shape[B.dim() - l2:]),
                           levi_civita(A.dtype))
    else:
        out = free_a + free_b
        spec = f"{lead}{''.join(a_idx)},{lead}{''.join(b_idx)}->{lead}{''.join(out)}"
        lead_shape = A.shape[: A.dim() - l1]
        res = torch.einsum(spec, A.reshape(-1, *A.shape[A.dim() - l1:]), B.reshape(-1, *B.shape[B.dim() - l2:]))
    return stf(res.reshape(*lead_shape, *([3] * l3)), l3)


def edge_attr(r: torch.Tensor, l: int) -> torch.Tensor:
    """STF part of u^(x)l for every edge, [E] + [3] * l."""
    n = torch.linalg.norm(r, dim=-1)
    ok = n >= R_EPS
    u = torch.where(ok[:, None], r / torch.where(ok, n, torch.ones_like(n))[:, None], torch.zeros_like(r))
    if l == 0:
        return torch.ones(r.shape[0], dtype=r.dtype)
    T = u
    for _ in range(l - 1):
        T = T[..., None] * u.reshape(u.shape[0], *([1] * (T.dim() - 1)), 3)
    return stf(T, l)


@lru_cache(maxsize=None)
def _sph_tensors(l: int) -> np.ndarray:
    """[2l+1, 3^l]: the symmetric coefficient tensor of each real harmonic Y_lm written as a
    homogeneous polynomial of degree l (terms of degree l - 2j times (x^2 + y^2 + z^2)^j)."""
    idx = list(itertools.product(range(3), repeat=l))
    out = np.zeros((2 * l + 1, 3 ** l))
    for m, terms in enumerate(sh_mod.sh_monomials(l)):
        hom = {}
        for (px, py, pz), c in terms.items():
            j = (l - (px + py + pz)) // 2
            for a in range(j + 1):              # multinomial expansion of (x^2 + y^2 + z^2)^j
                for b in range(j - a + 1):
                    cc = j - a - b
                    coef = c * _multinomial(j, a, b, cc)
                    key = (px + 2 * a, py + 2 * b, pz + 2 * cc)
                    hom[key] = hom.get(key, 0.0) + coef
        for i, t in enumerate(idx):
            cnt = (t.count(0), t.count(1), t.count(2))
            if cnt in hom:
                out[m, i] = hom[cnt] / _multinomial(l, *cnt)
    return out


def _multinomial(n: int, *ks: int) -> float:
    d = 1
    for k in ks:
        d *= factorial(k)
    return factorial(n) / d


def to_spherical(A: torch.Tensor, l: int) -> torch.Tensor:
    """Spherical components s_m = <T_lm, A> of STF tensors (trailing l indices): the map
    under which edge_attr(r, l) becomes Y_l(r) and rotations act by the Wigner matrices."""
    lead = A.shape[: A.dim() - l]
    T = torch.from_numpy(_sph_tensors(l)).to(A.dtype)
    return A.reshape(*lead, 3 ** l) @ T.T


class OracleCartTP:
    """Edge convolution with Cartesian couplings on the spherical oracle's path list."""

    def __init__(self, irreps_in: str, sh_lmax: int, irreps_out: str, C: int):
        self.paths = paths_mod.enumerate_paths(irreps_in, sh_lmax, irreps_out)
        self.ls_in = sorted({l for l, _ in paths_mod.parse_irreps(irreps_in)})
        self.ls_out = sorted({l for l, _ in paths_mod.parse_irreps(irreps_out)})
        self.sh_lmax, self.C = sh_lmax, C

    @property
    def P(self) -> int:
        return len(self.paths)

    def forward(self, row_ptr, src, r, x: dict, w) -> dict:
        """x: {l: [N, C] + [3] * l} STF tensors, w: [E, P, C]; returns {l3: [N, C] + [3] * l3}."""
        row_ptr = torch.as_tensor(np.asarray(row_ptr, dtype=np.int64))
        src = torch.as_tensor(np.asarray(src, dtype=np.int64))
        n = row_ptr.numel() - 1
        dst = torch.repeat_interleave(torch.arange(n), row_ptr[1:] - row_ptr[:-1])
        r = torch.as_tensor(r, dtype=torch.float64)
        w = torch.as_tensor(w, dtype=torch.float64)
        Y = {l: edge_attr(r, l) for l in range(self.sh_lmax + 1)}
        out = {l: torch.zeros(n, self.C, *([3] * l), dtype=torch.float64) for l in self.ls_out}
        for p, (l1, l2, l3) in enumerate(self.paths):
            xa = x[l1][src]                                           # [E, C] + [3] * l1
            yb = Y[l2].reshape(-1, 1, *([3] * l2)).expand(-1, self.C, *([3] * l2))
            msg = couple(xa, yb, l1, l2, l3) * w[:, p, :].reshape(-1, self.C, *([1] * l3))
            out[l3] = out[l3].index_add(0, dst, msg)
        return out

    def backward(self, row_ptr, src, r, x: dict, w, g: dict) -> dict:
        """VJP for the cotangent g ({l3: like out}): grad_x {l}, grad_w [E, P, C], grad_r [E, 3]."""
        xs = {l: torch.as_tensor(v, dtype=torch.float64).clone().requires_grad_(True) for l, v in x.items()}
        wt = torch.as_tensor(w, dtype=torch.float64).clone().requires_grad_(True)
        rt = torch.as_tensor(r, dtype=torch.float64).clone().requires_grad_(True)
        out = self.forward(row_ptr, src, rt, xs, wt)
        loss = sum((out[l] * torch.as_tensor(g[l], dtype=torch.float64)).sum() for l in out)
        grads = torch.autograd.grad(loss, [*xs.values(), wt, rt], allow_unused=True)
        gx = {l: (gr if gr is not None else torch.zeros_like(xs[l])) for l, gr in zip(xs, grads[: len(xs)])}
        return {"grad_x": gx, "grad_w": grads[len(xs)], "grad_r": grads[len(xs) + 1]}
