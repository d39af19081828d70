"""Pins of the oracle's tensor product, VJP and reverse grouping (oracle/__init__.py, etp_oracle.c).

Each test checks the FP64 oracle against something other than itself: hand closed
forms (l <= 1), a dense brute-force sum written independently in Python,
rotation equivariance, central finite differences, linearity, edge duplication,
and the special cases (empty rows, isolated sources, sampled outputs).
"""
import numpy as np
import pytest

import oracle
import workloads
from oracle import cg, sh


@pytest.fixture(scope="module")
def tiny():
    return workloads.make("tiny")


def _f64(wl):
    return wl.x.astype(np.float64), wl.w.astype(np.float64), wl.g.astype(np.float64)


def _dst(row_ptr):
    return np.repeat(np.arange(len(row_ptr) - 1), np.diff(row_ptr))


def test_closed_form_l1(tiny, oracle_built):
    """out_0 = w000 x0 + w110 (x1 . Y1)/sqrt3 ;  out_1 = w011 x0 Y1 + w101 x1 + w111 (x1 x Y1)/sqrt2."""
    tp = oracle.OracleTP("0+1", 1, "0+1", tiny.C)
    assert tp.paths == [(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 0), (1, 1, 1)]
    x, w, _ = _f64(tiny)
    out = tp.forward(tiny.row_ptr, tiny.src, tiny.r, x, w)
    want = np.zeros_like(out)
    dst = _dst(tiny.row_ptr)
    for e in range(tiny.E):
        i, j = dst[e], tiny.src[e]
        u = tiny.r[e].astype(np.float64)
        u = u / np.linalg.norm(u)
        Y1 = np.sqrt(3.0) * np.array([u[1], u[2], u[0]])   # components m = -1, 0, 1
        x0, x1 = x[j, 0], x[j, 1:4]                         # [C], [3, C]
        we = w[e]
        want[i, 0] += we[0] * x0 + we[3] * np.einsum("mc,m->c", x1, Y1) / np.sqrt(3)
        cross = np.stack([x1[1] * Y1[2] - x1[2] * Y1[1],
                          x1[2] * Y1[0] - x1[0] * Y1[2],
                          x1[0] * Y1[1] - x1[1] * Y1[0]])
        want[i, 1:4] += we[1] * x0[None, :] * Y1[:, None] + we[2] * x1 + we[4] * cross / np.sqrt(2)
    assert np.allclose(out, want, atol=1e-12)


def _brute(tp, wl, x, w, g):
    """Dense sum over all (i, j) pairs with a dense adjacency, dense CG blocks, Python loops."""
    N, E, C = wl.N, wl.E, wl.C
    dst = _dst(wl.row_ptr)
    edge_of = {}
    for e in range(E):
        edge_of[(int(dst[e]), int(wl.src[e]))] = e
    assert len(edge_of) == E, "brute force needs a simple graph"
    Y = sh.sh(tp.sh_lmax, wl.r)
    dY = sh.sh_grad(tp.sh_lmax, wl.r)
    out = np.zeros((N, tp.d_out, C))
    gx = np.zeros((N, tp.d_in, C))
    gw = np.zeros((E, tp.P, C))
    gr = np.zeros((E, 3))
    for i in range(N):
        for j in range(N):
            e = edge_of.get((i, j))
            if e is None:
                continue
            dLdY = np.zeros(Y.shape[1])
            for p, (l1, l2, l3) in enumerate(tp.paths):
                Cd = cg.real_cg(l1, l2, l3)
                a0, b0, o0 = l1 * l1, l2 * l2, l3 * l3
                for m1 in range(2 * l1 + 1):
                    for m2 in range(2 * l2 + 1):
                        for m3 in range(2 * l3 + 1):
                            c = Cd[m1, m2, m3]
                            if c == 0.0:
                                continue
                            xv, gv = x[j, a0 + m1], g[i, o0 + m3]
                            out[i, o0 + m3] += w[e, p] * c * Y[e, b0 + m2] * xv
                            gx[j, a0 + m1] += w[e, p] * c * Y[e, b0 + m2] * gv
                            gw[e, p] += c * Y[e, b0 + m2] * xv * gv
                            dLdY[b0 + m2] += np.sum(w[e, p] * c * xv * gv)
            gr[e] = dLdY @ dY[e]
    return out, gx, gw, gr


def test_brute_force_dense_sum(tiny, oracle_built):
    tp = oracle.OracleTP("0..1", 1, "0..1", tiny.C)
    x, w, g = _f64(tiny)
    out_b, gx_b, gw_b, gr_b = _brute(tp, tiny, x, w, g)
    out = tp.forward(tiny.row_ptr, tiny.src, tiny.r, x, w)
    res = tp.backward(tiny.row_ptr, tiny.src, tiny.r, x, w, g)
    assert np.allclose(out, out_b, atol=1e-12)
    assert np.allclose(res["grad_x"], gx_b, atol=1e-12)
    assert np.allclose(res["grad_w"], gw_b, atol=1e-12)
    assert np.allclose(res["grad_r"], gr_b, atol=1e-12)


def _small_l3(seed=11, n=12, e=60, C=3, irreps="0..3"):
    rng = np.random.default_rng(seed)
    P = len(oracle.paths.enumerate_paths(irreps, 3, irreps))
    wl = workloads.random_graph(rng, n, e, 3, C, P)
    return wl, P


def test_brute_force_l3_simple_graph(oracle_built):
    rng = np.random.default_rng(21)
    n, C = 6, 2
    pairs = [(i, j) for i in range(n) for j in range(n) if i != j and rng.random() < 0.5]
    dst = np.array([p[0] for p in pairs])
    src = np.array([p[1] for p in pairs])
    row_ptr, src_s, order = workloads.csr_from_pairs(n, dst, src)
    tp = oracle.OracleTP("0..3", 3, "0..3", C)
    E = len(src_s)
    wl = workloads.Workload("t", 3, C, tp.P, row_ptr, src_s, rng.standard_normal((E, 3)),
                            rng.standard_normal((n, 16, C)), rng.standard_normal((E, tp.P, C)),
                            rng.standard_normal((n, 16, C)))
    out_b, gx_b, gw_b, gr_b = _brute(tp, wl, wl.x, wl.w, wl.g)
    out = tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w)
    res = tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g)
    for a, b in [(out, out_b), (res["grad_x"], gx_b), (res["grad_w"], gw_b), (res["grad_r"], gr_b)]:
        assert np.allclose(a, b, atol=1e-11)


def _rotate_features(x, R, lmax):
    y = np.empty_like(x)
    for l in range(lmax + 1):
        D = cg.wigner_d(l, R, seed=4242)
        y[:, l * l:(l + 1) ** 2] = np.einsum("ab,nbc->nac", D, x[:, l * l:(l + 1) ** 2])
    return y


@pytest.mark.parametrize("irreps", ["0..3", "0e+1o+2e+3o"])
def test_rotation_equivariance(irreps, oracle_built):
    wl, P = _small_l3(irreps=irreps)
    tp = oracle.OracleTP(irreps, 3, irreps, wl.C)
    x, w, g = (a.astype(np.float64) for a in (wl.x, wl.w, wl.g))
    r = wl.r.astype(np.float64)
    R = cg.random_rotation(np.random.default_rng(99))
    out = tp.forward(wl.row_ptr, wl.src, r, x, w)
    out_rot = tp.forward(wl.row_ptr, wl.src, r @ R.T, _rotate_features(x, R, 3), w)
    scale = np.max(np.abs(out))
    assert np.max(np.abs(out_rot - _rotate_features(out, R, 3))) <= 1e-12 * scale
    b = tp.backward(wl.row_ptr, wl.src, r, x, w, g)
    br = tp.backward(wl.row_ptr, wl.src, r @ R.T, _rotate_features(x, R, 3), w, _rotate_features(g, R, 3))
    assert np.max(np.abs(br["grad_x"] - _rotate_features(b["grad_x"], R, 3))) <= 1e-12 * np.max(np.abs(b["grad_x"]))
    assert np.max(np.abs(br["grad_w"] - b["grad_w"])) <= 1e-12 * np.max(np.abs(b["grad_w"]))
    assert np.max(np.abs(br["grad_r"] - b["grad_r"] @ R.T)) <= 1e-11 * np.max(np.abs(b["grad_r"]))


def test_inversion_parity_o3(oracle_built):
    """With natural parities, r -> -r and x_l -> (-1)^l x_l maps out_l -> (-1)^l out_l."""
    irreps = "0e+1o+2e+3o"
    wl, P = _small_l3(irreps=irreps)
    tp = oracle.OracleTP(irreps, 3, irreps, wl.C)
    x, w = wl.x.astype(np.float64), wl.w.astype(np.float64)
    sgn = np.concatenate([np.full(2 * l + 1, (-1.0) ** l) for l in range(4)])[None, :, None]
    out = tp.forward(wl.row_ptr, wl.src, wl.r, x, w)
    out_inv = tp.forward(wl.row_ptr, wl.src, -wl.r.astype(np.float64), x * sgn, w)
    assert np.allclose(out_inv, out * sgn, atol=1e-12)


@pytest.mark.parametrize("which", ["tiny", "l3"])
def test_vjp_by_central_differences(which, tiny, oracle_built):
    if which == "tiny":
        wl, irreps, lmax = tiny, "0..1", 1
    else:
        wl, _ = _small_l3(seed=5, n=8, e=24, C=2)
        irreps, lmax = "0..3", 3
    tp = oracle.OracleTP(irreps, lmax, irreps, wl.C)
    x, w, g = (a.astype(np.float64) for a in (wl.x, wl.w, wl.g))
    r = wl.r.astype(np.float64)
    loss = lambda xx, ww, rr: np.sum(tp.forward(wl.row_ptr, wl.src, rr, xx, ww) * g)
    b = tp.backward(wl.row_ptr, wl.src, r, x, w, g)
    rng = np.random.default_rng(17)
    h = 1e-6
    for name, base, grad in [("x", x, b["grad_x"]), ("w", w, b["grad_w"]), ("r", r, b["grad_r"])]:
        for _ in range(3):
            d = rng.standard_normal(base.shape)
            args = {"x": x, "w": w, "r": r}
            args_p, args_m = dict(args), dict(args)
            args_p[name] = base + h * d
            args_m[name] = base - h * d
            fd = (loss(args_p["x"], args_p["w"], args_p["r"]) - loss(args_m["x"], args_m["w"], args_m["r"])) / (2 * h)
            an = np.sum(grad * d)
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
    # single entries of grad_r as well
    for e in [0, wl.E // 2, wl.E - 1]:
        for a in range(3):
            rp, rm = r.copy(), r.copy()
            rp[e, a] += h
            rm[e, a] -= h
            fd = (loss(x, w, rp) - loss(x, w, rm)) / (2 * h)
            assert abs(fd - b["grad_r"][e, a]) <= 1e-6 * max(1.0, abs(fd))
    # derivative through the direction only: r_e . grad_r[e] = 0
    assert np.allclose(np.sum(r * b["grad_r"], axis=1), 0.0, atol=1e-9 * np.max(np.abs(b["grad_r"])))


def test_linearity_and_edge_duplication(tiny, oracle_built):
    tp = oracle.OracleTP("0..1", 1, "0..1", tiny.C)
    x, w, _ = _f64(tiny)
    f = lambda xx, ww: tp.forward(tiny.row_ptr, tiny.src, tiny.r, xx, ww)
    rng = np.random.default_rng(8)
    x2, w2 = rng.standard_normal(x.shape), rng.standard_normal(w.shape)
    assert np.allclose(f(2.5 * x + x2, w), 2.5 * f(x, w) + f(x2, w), atol=1e-12)
    assert np.allclose(f(x, w - 3 * w2), f(x, w) - 3 * f(x, w2), atol=1e-12)
    # every edge twice (rows keep sources ascending) doubles the output
    dst = _dst(tiny.row_ptr)
    dd, ss = np.concatenate([dst, dst]), np.concatenate([tiny.src, tiny.src])
    row_ptr2, src2, order = workloads.csr_from_pairs(tiny.N, dd, ss)
    eid = np.concatenate([np.arange(tiny.E), np.arange(tiny.E)])[order]
    out2 = tp.forward(row_ptr2, src2, tiny.r[eid], x, w[eid])
    assert np.allclose(out2, 2 * f(x, w), atol=1e-12)


def test_empty_rows_isolated_sources_and_sampling(oracle_built):
    wl, P = _small_l3(seed=3, n=10, e=40, C=4)
    tp = oracle.OracleTP("0..3", 3, "0..3", wl.C)
    out = tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w)
    empty = np.flatnonzero(np.diff(wl.row_ptr) == 0)
    assert len(empty) >= 1 and np.all(out[empty] == 0.0)
    b = tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g)
    iso = np.setdiff1d(np.arange(wl.N), wl.src)
    assert len(iso) >= 1 and np.all(b["grad_x"][iso] == 0.0)
    rows = np.array([7, 2, 2, 9])
    assert np.array_equal(tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, rows=rows), out[rows])
    edges = np.array([39, 0, 17])
    nodes = np.array([4, 1])
    bs = tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g, nodes=nodes, edges=edges)
    assert np.array_equal(bs["grad_x"], b["grad_x"][nodes])
    assert np.array_equal(bs["grad_w"], b["grad_w"][edges])
    assert np.array_equal(bs["grad_r"], b["grad_r"][edges])
    # fp32 inputs take the float entry points and agree with the double ones
    assert np.allclose(tp.forward(wl.row_ptr, wl.src, wl.r, wl.x.astype(np.float64), wl.w.astype(np.float64)),
                       out, atol=1e-13)


def test_no_edges(oracle_built):
    tp = oracle.OracleTP("0..2", 2, "0..2", 4)
    n = 5
    row_ptr = np.zeros(n + 1, dtype=np.int32)
    src = np.zeros(0, dtype=np.int32)
    x = np.ones((n, 9, 4), np.float32)
    w = np.zeros((0, tp.P, 4), np.float32)
    out = tp.forward(row_ptr, src, np.zeros((0, 3), np.float32), x, w)
    assert out.shape == (n, 9, 4) and not out.any()
    b = tp.backward(row_ptr, src, np.zeros((0, 3), np.float32), x, w, x)
    assert not b["grad_x"].any() and b["grad_w"].shape == (0, tp.P, 4) and b["grad_r"].shape == (0, 3)


def test_reverse_csr_brute_force():
    rng = np.random.default_rng(1)
    for n, e in [(1, 0), (1, 5), (7, 0), (9, 50), (40, 300)]:
        dst = rng.integers(0, n, e)
        src = rng.integers(0, n, e)
        row_ptr, s, _ = workloads.csr_from_pairs(n, dst, src)
        rev_ptr, rev_perm, d = oracle.reverse_csr(n, row_ptr, s)
        want_ptr, want_perm = [0], []
        for j in range(n):
            for k in range(e):
                if s[k] == j:
                    want_perm.append(k)
            want_ptr.append(len(want_perm))
        assert rev_ptr.tolist() == want_ptr and rev_perm.tolist() == want_perm
        want_d = []
        for i in range(n):
            want_d += [i] * int(row_ptr[i + 1] - row_ptr[i])
        assert d.tolist() == want_d


@pytest.mark.parametrize("mistake", ["flip_sign", "drop_entry", "mirror_m1", "shift_sh", "swap_path_weights"])
def test_pins_catch_planted_mistakes(mistake, oracle_built):
    """A corrupted copy of the oracle's tables must fail the equivariance pin or the closed form."""
    irreps = "0..3"
    wl, P = _small_l3(seed=31, n=9, e=30, C=2)
    good = oracle.OracleTP(irreps, 3, irreps, wl.C)
    bad = oracle.OracleTP(irreps, 3, irreps, wl.C)
    k = int(np.flatnonzero(bad.path_off[1:] - bad.path_off[:-1] > 3)[5])   # some path with several entries
    lo, hi = bad.path_off[k], bad.path_off[k + 1]
    if mistake == "flip_sign":
        bad.cg_val[lo + 1] *= -1
    elif mistake == "drop_entry":
        bad.cg_val[lo + 1] = 0.0
    elif mistake == "mirror_m1":
        # x read at -m1 instead of m1 inside one l1 = 2 block
        k = next(q for q, (a, b, c) in enumerate(bad.paths) if (a, b, c) == (2, 1, 2))
        lo, hi = bad.path_off[k], bad.path_off[k + 1]
        bad.cg_in[lo:hi] = 4 + (4 - (bad.cg_in[lo:hi] - 4))
    elif mistake == "shift_sh":
        l2 = bad.paths[k][1]
        bad.cg_sh[lo:hi] = l2 * l2 + (bad.cg_sh[lo:hi] - l2 * l2 + 1) % (2 * l2 + 1)
    elif mistake == "swap_path_weights":
        bad.cg_val = bad.cg_val.copy()
        a, b = bad.path_off[k], bad.path_off[k + 1]
        bad.cg_val[a:b] = bad.cg_val[a:b][::-1]
    x, w = wl.x.astype(np.float64), wl.w.astype(np.float64)
    r = wl.r.astype(np.float64)
    R = cg.random_rotation(np.random.default_rng(5))

    def equiv_err(tp):
        out = tp.forward(wl.row_ptr, wl.src, r, x, w)
        out_rot = tp.forward(wl.row_ptr, wl.src, r @ R.T, _rotate_features(x, R, 3), w)
        return np.max(np.abs(out_rot - _rotate_features(out, R, 3))) / np.max(np.abs(out))

    assert equiv_err(good) < 1e-12
    assert equiv_err(bad) > 1e-6, mistake
