"""FP64 CPU oracle for the edge-wise equivariant tensor product, its VJP and the
VJP of its VJP (double backward).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import, call, link or execute anything under
``oracle/``. The CUDA library never does, and the two share no code, header or
table: the oracle builds its own spherical harmonics (``sh.py``, textbook
polynomial definition), its own coupling tensors (``cg.py``, invariance
construction), its own path list (``paths.py``), its own reverse grouping of
edges (``reverse_csr`` below) and runs its own FP64 loops (``etp_oracle.c``).

Every function here is pinned by ``tests/test_oracle_*.py`` against closed
forms, library routines, invariants, finite differences and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

from . import cg as cg_mod
from . import paths as paths_mod
from . import sh as sh_mod
from .forces import assemble_forces  # noqa: F401  (forces and per-atom virials from dE/dr)
from . import radial  # noqa: F401  (radial-weight MLP of the edge length and its VJP)
from . import cartesian  # noqa: F401  (the same edge convolution with Cartesian couplings)
from . import nodelocal  # noqa: F401  (the node-local product, spherical and Cartesian)

_HERE = os.path.dirname(os.path.abspath(__file__))
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libetp_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C loops (gcc, OpenMP, -O2, no fast-math) into oracle/_build."""
    srcs = [os.path.join(_HERE, "etp_oracle.c"), os.path.join(_HERE, "etp_oracle_impl.h")]
    if not force and os.path.exists(_LIB_PATH):
        if os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(s) for s in srcs):
            return _LIB_PATH
    os.makedirs(_BUILD, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-ffp-contract=off", srcs[0], "-o", tmp])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB_PATH)
        _lib.oracle_num_threads.restype = ctypes.c_int
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def reverse_csr(n_nodes: int, row_ptr: np.ndarray, src: np.ndarray):
    """Edges grouped by source, stable in edge id; and the destination of every edge.

    rev_ptr[j]..rev_ptr[j+1] indexes rev_perm, which lists the edges with source
    j in increasing edge id; dst[e] is the CSR row that holds e.
    """
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    src = np.asarray(src, dtype=np.int64)
    counts = np.bincount(src, minlength=n_nodes)
    rev_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rev_perm = np.argsort(src, kind="stable").astype(np.int32)
    dst = np.repeat(np.arange(n_nodes), np.diff(row_ptr)).astype(np.int32)
    return rev_ptr, rev_perm, dst


@dataclass
class OracleTP:
    """Tensor product of node irreps with edge harmonics, per-edge weights, segment sum."""

    irreps_in: str
    sh_lmax: int
    irreps_out: str
    C: int
    paths: list = field(init=False)

    def __post_init__(self):
        self.paths = paths_mod.enumerate_paths(self.irreps_in, self.sh_lmax, self.irreps_out)
        ins = paths_mod.parse_irreps(self.irreps_in)
        outs = paths_mod.parse_irreps(self.irreps_out)
        self.in_off, self.d_in = paths_mod.block_offsets(ins)
        self.out_off, self.d_out = paths_mod.block_offsets(outs)
        self.d_sh = (self.sh_lmax + 1) ** 2
        path_off, a, b, o, v = [0], [], [], [], []
        for (l1, l2, l3) in self.paths:
            for m1, m2, m3, val in cg_mod.nnz_list(l1, l2, l3):
                a.append(self.in_off[l1] + m1)
                b.append(l2 * l2 + m2)
                o.append(self.out_off[l3] + m3)
                v.append(val)
            path_off.append(len(v))
        self.path_off = np.asarray(path_off, dtype=np.int32)
        self.cg_in = np.asarray(a, dtype=np.int32)
        self.cg_sh = np.asarray(b, dtype=np.int32)
        self.cg_out = np.asarray(o, dtype=np.int32)
        self.cg_val = np.asarray(v, dtype=np.float64)

    @property
    def P(self) -> int:
        return len(self.paths)

    @property
    def nnz(self) -> int:
        return len(self.cg_val)

    def _tables(self):
        return (ctypes.c_int(self.C), ctypes.c_int(self.d_in), ctypes.c_int(self.d_sh),
                ctypes.c_int(self.d_out), ctypes.c_int(self.P), _p(self.path_off),
                _p(self.cg_in), _p(self.cg_sh), _p(self.cg_out), _p(self.cg_val))

    @staticmethod
    def _kind(*arrs):
        dt = {a.dtype for a in arrs}
        if dt == {np.dtype(np.float32)}:
            return "_f32"
        if dt == {np.dtype(np.float64)}:
            return "_f64"
        raise TypeError(f"x, w, g must all be float32 or all float64, got {dt}")

    def _check(self, n_nodes, row_ptr, src, r, x, w):
        E = len(src)
        assert row_ptr.shape == (n_nodes + 1,) and row_ptr[0] == 0 and row_ptr[-1] == E
        assert r.shape == (E, 3)
        assert x.shape == (n_nodes, self.d_in, self.C)
        assert w.shape == (E, self.P, self.C)

    def forward(self, row_ptr, src, r, x, w, rows=None) -> np.ndarray:
        """out[rows] as FP64, shape [len(rows), d_out, C] (all rows if None)."""
        lib = _load()
        n = len(row_ptr) - 1
        row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
        src = np.ascontiguousarray(src, dtype=np.int32)
        x, w = np.ascontiguousarray(x), np.ascontiguousarray(w)
        self._check(n, row_ptr, src, r, x, w)
        rows = np.arange(n, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
        Y = np.ascontiguousarray(sh_mod.sh(self.sh_lmax, r))
        out = np.zeros((len(rows), self.d_out, self.C), dtype=np.float64)
        fn = getattr(lib, "oracle_forward" + self._kind(x, w))
        fn(ctypes.c_int64(len(rows)), _p(rows), _p(row_ptr), _p(src), *self._tables(),
           _p(Y), _p(x), _p(w), _p(out))
        return out

    def backward(self, row_ptr, src, r, x, w, g, nodes=None, edges=None,
                 want=("x", "w", "r")) -> dict:
        """grad_x[nodes] [n, d_in, C], grad_w[edges] [m, P, C], grad_r[edges] [m, 3] in FP64."""
        lib = _load()
        n = len(row_ptr) - 1
        row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
        src = np.ascontiguousarray(src, dtype=np.int32)
        x, w, g = np.ascontiguousarray(x), np.ascontiguousarray(w), np.ascontiguousarray(g)
        self._check(n, row_ptr, src, r, x, w)
        assert g.shape == (n, self.d_out, self.C)
        kind = self._kind(x, w, g)
        rev_ptr, rev_perm, dst = reverse_csr(n, row_ptr, src)
        Y = np.ascontiguousarray(sh_mod.sh(self.sh_lmax, r))
        res = {}
        if "x" in want:
            nodes_ = np.arange(n, dtype=np.int64) if nodes is None else np.ascontiguousarray(nodes, dtype=np.int64)
            gx = np.zeros((len(nodes_), self.d_in, self.C), dtype=np.float64)
            getattr(lib, "oracle_grad_x" + kind)(
                ctypes.c_int64(len(nodes_)), _p(nodes_), _p(rev_ptr), _p(rev_perm), _p(dst),
                *self._tables(), _p(Y), _p(w), _p(g), _p(gx))
            res["grad_x"] = gx
        if "w" in want or "r" in want:
            E = len(src)
            edges_ = np.arange(E, dtype=np.int64) if edges is None else np.ascontiguousarray(edges, dtype=np.int64)
            dY = np.ascontiguousarray(sh_mod.sh_grad(self.sh_lmax, r)) if "r" in want else None
            gw = np.zeros((len(edges_), self.P, self.C), dtype=np.float64) if "w" in want else None
            gr = np.zeros((len(edges_), 3), dtype=np.float64) if "r" in want else None
            if dY is None:
                dY = np.zeros((1,), dtype=np.float64)
            getattr(lib, "oracle_grad_wr" + kind)(
                ctypes.c_int64(len(edges_)), _p(edges_), _p(src), _p(dst), *self._tables(),
                _p(Y), _p(dY), _p(x), _p(w), _p(g), _p(gw), _p(gr))
            if gw is not None:
                res["grad_w"] = gw
            if gr is not None:
                res["grad_r"] = gr
        return res


    def double_backward(self, row_ptr, src, r, x, w, g, gg_x=None, gg_w=None, gg_r=None) -> dict:
        """VJP of the VJP: the gradients of <gg_x, grad_x> + <gg_w, grad_w> + <gg_r, grad_r>
        with respect to g, x, w and r, where (grad_x, grad_w, grad_r) = VJP(x, w, r; g).

        Force-loss training differentiates the forces (built from grad_r) with respect to
        the parameters, which takes this second-order product; FlashCart times it beside the
        forward and the VJP ("FlashCart 如何让等变原子间势更快更准?", section
        "生成内核在高阶下胜过球谐基线"). Written out from the definition: the tensor product
        is linear in each of x, w, g and Y, so every term is one of the first-order loops
        with one input replaced by its cotangent. With Ydot[e] = dY/dr[e] . gg_r[e] (the
        directional derivative of the harmonics) and Hg[e] = d2Y/dr2[e] . gg_r[e]:

            grad_g = fwd(x <- gg_x) + fwd(w <- gg_w) + fwd(Y <- Ydot)
            grad_x = vjp_x(w <- gg_w) + vjp_x(Y <- Ydot)
            grad_w = vjp_w(x <- gg_x) + vjp_w(Y <- Ydot)
            grad_r = vjp_r(x <- gg_x) + vjp_r(w <- gg_w) + vjp_r(dY/dr <- Hg)

        A cotangent given as None is zero. Everything in FP64; returns grad_g [N, d_out, C],
        grad_x [N, d_in, C], grad_w [E, P, C], grad_r [E, 3].
        """
        lib = _load()
        f64 = lambda a: np.ascontiguousarray(a, dtype=np.float64)
        n = len(row_ptr) - 1
        row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
        src = np.ascontiguousarray(src, dtype=np.int32)
        r, x, w, g = f64(r), f64(x), f64(w), f64(g)
        self._check(n, row_ptr, src, r, x, w)
        assert g.shape == (n, self.d_out, self.C)
        E = len(src)
        rev_ptr, rev_perm, dst = reverse_csr(n, row_ptr, src)
        nodes = np.arange(n, dtype=np.int64)
        edges = np.arange(E, dtype=np.int64)
        Y = f64(sh_mod.sh(self.sh_lmax, r))
        dY = f64(sh_mod.sh_grad(self.sh_lmax, r))
        none = np.zeros((1,), dtype=np.float64)

        def fwd(Ya, xa, wa):
            out = np.zeros((n, self.d_out, self.C), dtype=np.float64)
            lib.oracle_forward_f64(ctypes.c_int64(n), _p(nodes), _p(row_ptr), _p(src), *self._tables(),
                                   _p(Ya), _p(xa), _p(wa), _p(out))
            return out

        def vjp_x(Ya, wa):
            gx = np.zeros((n, self.d_in, self.C), dtype=np.float64)
            lib.oracle_grad_x_f64(ctypes.c_int64(n), _p(nodes), _p(rev_ptr), _p(rev_perm), _p(dst), *self._tables(),
                                  _p(Ya), _p(wa), _p(g), _p(gx))
            return gx

        def vjp_wr(Ya, dYa, xa, wa, want_w, want_r):
            gw = np.zeros((E, self.P, self.C), dtype=np.float64) if want_w else None
            gr = np.zeros((E, 3), dtype=np.float64) if want_r else None
            lib.oracle_grad_wr_f64(ctypes.c_int64(E), _p(edges), _p(src), _p(dst), *self._tables(),
                                   _p(Ya), _p(dYa if dYa is not None else none), _p(xa), _p(wa), _p(g), _p(gw), _p(gr))
            return gw, gr

        res = {"grad_g": np.zeros((n, self.d_out, self.C)), "grad_x": np.zeros((n, self.d_in, self.C)),
               "grad_w": np.zeros((E, self.P, self.C)), "grad_r": np.zeros((E, 3))}
        if gg_x is not None:
            gg_x = f64(gg_x)
            assert gg_x.shape == x.shape
            res["grad_g"] += fwd(Y, gg_x, w)
            gw, gr = vjp_wr(Y, dY, gg_x, w, True, True)
            res["grad_w"] += gw
            res["grad_r"] += gr
        if gg_w is not None:
            gg_w = f64(gg_w)
            assert gg_w.shape == w.shape
            res["grad_g"] += fwd(Y, x, gg_w)
            res["grad_x"] += vjp_x(Y, gg_w)
            res["grad_r"] += vjp_wr(Y, dY, x, gg_w, False, True)[1]
        if gg_r is not None:
            gg_r = f64(gg_r)
            assert gg_r.shape == (E, 3)
            Ydot = f64(np.einsum("eka,ea->ek", dY, gg_r))
            Hg = f64(np.einsum("ekab,eb->eka", sh_mod.sh_hess(self.sh_lmax, r), gg_r))
            res["grad_g"] += fwd(Ydot, x, w)
            res["grad_x"] += vjp_x(Ydot, w)
            res["grad_w"] += vjp_wr(Ydot, None, x, w, True, False)[0]
            res["grad_r"] += vjp_wr(Y, Hg, x, w, False, True)[1]
        return res
