"""The library's layout of Cartesian features: a rank-l STF tensor held by its 2l + 1
entries with at most one z index (x^l, x^(l-1) y, .., y^l, x^(l-1) z, .., y^(l-1) z), mapped
to and from the oracle's full 3^l tensors by the tests' own expansion (STF completion) and
entry picks. Test infrastructure; no GPU needed."""
import itertools

import numpy as np
import torch

from oracle import cartesian as ct


def counts(l):
    return [(l - b, b, 0) for b in range(l + 1)] + [(l - 1 - b, b, 1) for b in range(l)]


def pick(l):
    """S [2l+1, 3^l]: the independent entries of a full rank-l tensor."""
    if l == 0:
        return np.ones((1, 1))
    pos = {t: i for i, t in enumerate(itertools.product(range(3), repeat=l))}
    S = np.zeros((2 * l + 1, 3 ** l))
    for i, (a, b, c) in enumerate(counts(l)):
        S[i, pos[(0,) * a + (1,) * b + (2,) * c]] = 1.0
    return S


def expand(l):
    """E [3^l, 2l+1]: the STF tensor with the given independent entries (S E = I)."""
    if l == 0:
        return np.ones((1, 1))
    u, s, _ = np.linalg.svd(ct.stf_projector(l))
    Q = u[:, s > 0.5]
    return Q @ np.linalg.inv(pick(l) @ Q)


def to_full(a, L):
    """[N, (L+1)^2, C] independent components -> {l: [N, C] + [3] * l} full tensors."""
    out = {}
    for l in range(L + 1):
        blk = a[:, l * l:(l + 1) ** 2, :].astype(np.float64)             # [N, 2l+1, C]
        full = np.einsum("fi,nic->ncf", expand(l), blk)
        out[l] = torch.from_numpy(full.reshape(a.shape[0], a.shape[2], *([3] * l)) if l else full[..., 0])
    return out


def from_full(d, L, op):
    """{l: [N, C] + [3]*l} -> [N, (L+1)^2, C] with op(l) ([2l+1, 3^l]) applied to each tensor."""
    blocks = []
    for l in range(L + 1):
        t = d[l].detach().numpy().reshape(d[l].shape[0], d[l].shape[1], -1)
        blocks.append(np.einsum("if,ncf->nic", op(l), t))
    return np.concatenate(blocks, axis=1)


def coupling_table(l1, l2, l3):
    """T [2l1+1, 2l2+1, 2l3+1]: the oracle's Cartesian coupling of path (l1, l2, l3) in the
    library's independent components, out[i3] = sum T[i1, i2, i3] A[i1] B[i2] (A, B expanded
    to full STF tensors, the result's independent entries picked)."""
    d1, d2 = 2 * l1 + 1, 2 * l2 + 1
    T = np.zeros((d1, d2, 2 * l3 + 1))
    for i in range(d1):
        for j in range(d2):
            a = torch.from_numpy(expand(l1)[:, i].reshape((1,) + (3,) * l1))
            b = torch.from_numpy(expand(l2)[:, j].reshape((1,) + (3,) * l2))
            full = ct.couple(a, b, l1, l2, l3).reshape(-1).numpy()
            T[i, j] = pick(l3) @ full
    return T
