"""GPU parity of the VJP of the VJP (etp_double_backward) against the FP64 oracle
(OracleTP.double_backward): gradients of <gg_x, grad_x> + <gg_w, grad_w> +
<gg_r, grad_r> with respect to grad_out, x, w and r. Tolerance: the VJP's 1e-4
(max error over max |oracle|, per output). Full-size graphs are checked on sampled
destination rows, source nodes and edges, each from a sub-graph that holds every
edge the sampled outputs depend on."""
import numpy as np
import pytest
import torch

import cg_tensor_products_b200 as etp
import oracle
import workloads
from cg_tensor_products_b200 import build as etp_build
from gpu_helpers import VJP_TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    etp_build.build()
    oracle.build()


def _cotangents(wl, P, seed):
    rng = np.random.default_rng(seed)
    D = (wl.L + 1) ** 2
    ggx = rng.standard_normal((wl.N, D, wl.C), dtype=np.float32)
    ggw = rng.standard_normal((wl.E, P, wl.C), dtype=np.float32)
    ggw *= np.float32(1.0 / np.sqrt(P))
    ggr = rng.standard_normal((wl.E, 3), dtype=np.float32)
    return ggx, ggw, ggr


def _gpu(plan, wl, w, ggx, ggw, ggr, want=("g", "x", "w", "r")):
    d = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    rp, src = d(wl.row_ptr), d(wl.src)
    rev_ptr, rev_perm, dst = etp.build_reverse_csr(wl.N, rp, src)
    out = etp.double_backward(plan, rp, src, rev_ptr, rev_perm, dst, d(wl.r), d(wl.x), d(w), d(wl.g),
                              d(ggx), d(ggw), d(ggr), want=want)
    torch.cuda.synchronize()
    assert etp.device_fault() == 0
    return out


def _compare(out, ref, keys=("grad_g", "grad_x", "grad_w", "grad_r")):
    errs = {k: rel_err(out[k], ref[k]) for k in keys if k in out}
    assert all(v <= VJP_TOL for v in errs.values()), errs
    return errs


@pytest.mark.parametrize("L,o3,C,N,E", [(0, False, 8, 20, 300), (1, False, 8, 40, 700), (1, True, 32, 30, 900),
                                        (2, False, 64, 50, 1500), (2, True, 16, 30, 800), (2, False, 4, 17, 333),
                                        (3, False, 128, 40, 1200), (3, True, 64, 33, 1000), (3, False, 8, 20, 515)])
def test_every_spec_ragged_multigraph(L, o3, C, N, E):
    """Ragged random multigraphs (duplicate edges, an empty row, a source without
    edges, a zero-length edge) for every compiled specialisation."""
    rng = np.random.default_rng(L * 101 + C + E)
    wl = workloads.random_graph(rng, N, E, L, C, workloads.N_PATHS_SO3[L])
    irreps = "+".join(f"{l}{'e' if l % 2 == 0 else 'o'}" for l in range(L + 1)) if o3 else wl.irreps
    plan = etp.Plan(irreps, L, irreps, C)
    P = plan.n_paths
    w = (rng.standard_normal((E, P, C)) / np.sqrt(P)).astype(np.float32)
    wl.r[E // 3] = 0.0
    ggx, ggw, ggr = _cotangents(wl, P, 7)
    out = _gpu(plan, wl, w, ggx, ggw, ggr)
    tp = oracle.OracleTP(irreps, L, irreps, C)
    ref = tp.double_backward(wl.row_ptr, wl.src, wl.r, wl.x, w, wl.g, gg_x=ggx, gg_w=ggw, gg_r=ggr)
    _compare(out, ref)


@pytest.mark.parametrize("name", ["tiny", "water"])
def test_workload_full(name):
    wl = workloads.make(name)
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    ggx, ggw, ggr = _cotangents(wl, wl.P, 3)
    out = _gpu(plan, wl, wl.w, ggx, ggw, ggr)
    ref = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C).double_backward(
        wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g, gg_x=ggx, gg_w=ggw, gg_r=ggr)
    _compare(out, ref)


@pytest.mark.parametrize("cot", [("x",), ("w",), ("r",), ("x", "r")])
def test_single_cotangents_and_subsets(cot):
    """Each cotangent alone (the others NULL), and a subset of the outputs."""
    wl = workloads.make("tiny")
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    ggx, ggw, ggr = _cotangents(wl, wl.P, 5)
    ggx, ggw, ggr = (a if k in cot else None for a, k in ((ggx, "x"), (ggw, "w"), (ggr, "r")))
    tp = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C)
    ref = tp.double_backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g, gg_x=ggx, gg_w=ggw, gg_r=ggr)
    out = _gpu(plan, wl, wl.w, ggx, ggw, ggr)
    for k in ("grad_g", "grad_x", "grad_w", "grad_r"):
        assert rel_err(out[k], ref[k]) <= VJP_TOL, (k, cot)
    part = _gpu(plan, wl, wl.w, ggx, ggw, ggr, want=("x", "r"))
    assert "grad_g" not in part and "grad_w" not in part
    assert torch.equal(part["grad_x"], out["grad_x"]) and torch.equal(part["grad_r"], out["grad_r"])


def _sub(wl, keep_edge):
    """The graph restricted to the kept edges (same nodes, CSR by destination)."""
    dst = np.repeat(np.arange(wl.N), np.diff(wl.row_ptr))[keep_edge]
    counts = np.bincount(dst, minlength=wl.N)
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return row_ptr, wl.src[keep_edge], wl.r[keep_edge]


@pytest.mark.parametrize("name", ["micro_l3", "large"])
def test_full_size_sampled(name):
    wl = workloads.make(name)
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    ggx, ggw, ggr = _cotangents(wl, wl.P, 9)
    out = _gpu(plan, wl, wl.w, ggx, ggw, ggr)
    tp = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C)
    rng = np.random.default_rng(2)
    dst_all = np.repeat(np.arange(wl.N), np.diff(wl.row_ptr))
    rows = np.unique(np.concatenate([[0, wl.N - 1], rng.integers(0, wl.N, 24)]))
    nodes = np.unique(np.concatenate([[0, wl.N - 1], rng.integers(0, wl.N, 24)]))
    for key, sel, pick in (("grad_g", np.isin(dst_all, rows), rows), ("grad_x", np.isin(wl.src, nodes), nodes)):
        rp, sv, rv = _sub(wl, sel)
        ref = tp.double_backward(rp, sv, rv, wl.x, wl.w[sel], wl.g, gg_x=ggx, gg_w=ggw[sel], gg_r=ggr[sel])
        got = out[key][torch.from_numpy(pick).cuda()]
        assert rel_err(got, ref[key][pick]) <= VJP_TOL, key
        if key == "grad_g":  # per-edge outputs of the sampled rows' edges
            idx = torch.from_numpy(np.nonzero(sel)[0]).cuda()
            assert rel_err(out["grad_w"][idx], ref["grad_w"]) <= VJP_TOL
            assert rel_err(out["grad_r"][idx], ref["grad_r"]) <= VJP_TOL


@pytest.mark.parametrize("C", [32, 128])
def test_hub_rows_repeatable(C):
    """Hub rows cut across many tasks (grad_g and grad_x): oracle parity, and two runs
    agree bit for bit (partial rows summed in task order, no atomics)."""
    from gpu_helpers import hub_workload

    wl = hub_workload(np.random.default_rng(31), 2, C, 15, hub=6000, rest=1000)
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    ggx, ggw, ggr = _cotangents(wl, wl.P, 11)
    a = _gpu(plan, wl, wl.w, ggx, ggw, ggr)
    b = _gpu(plan, wl, wl.w, ggx, ggw, ggr)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    ref = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C).double_backward(
        wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g, gg_x=ggx, gg_w=ggw, gg_r=ggr)
    _compare(a, ref)
