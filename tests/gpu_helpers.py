"""Shared helpers of the GPU parity tests: move a workload to the device, run the
library through its binding, and compare with the FP64 oracle.

Error measure (per output tensor): max |gpu - oracle| / max |oracle| over the
compared entries; forward <= 1e-5, VJP <= 1e-4. Integer outputs: bit-exact.
"""
import numpy as np
import torch

import cg_tensor_products_b200 as etp
import oracle

FWD_TOL = 1e-5
VJP_TOL = 1e-4


def rel_err(gpu, ref) -> float:
    g = gpu.detach().cpu().numpy().astype(np.float64) if isinstance(gpu, torch.Tensor) else np.asarray(gpu)
    den = np.max(np.abs(ref)) if ref.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(g))) if g.size else 0.0
    return float(np.max(np.abs(g - ref)) / den)


def to_dev(wl, dev="cuda:0"):
    return {k: torch.from_numpy(np.ascontiguousarray(getattr(wl, k))).to(dev)
            for k in ("row_ptr", "src", "r", "x", "w", "g")}


def run_gpu(wl, irreps=None, with_dst=True, want=("x", "w", "r"), framed=False):
    """Forward, reverse CSR and VJP through the binding. framed: the edge frames
    are built once by etp_edge_frames and both kernels read them (r is then not
    passed to the kernels at all)."""
    irreps = irreps or wl.irreps
    plan = etp.Plan(irreps, wl.L, irreps, wl.C)
    t = to_dev(wl)
    frames = etp.edge_frames(plan, t["r"]) if framed else None
    r = None if framed else t["r"]
    out = etp.forward(plan, t["row_ptr"], t["src"], r, t["x"], t["w"], frames=frames)
    rev_ptr, rev_perm, dst = etp.build_reverse_csr(wl.N, t["row_ptr"], t["src"], with_dst=with_dst)
    gx, gw, gr = etp.backward(plan, t["row_ptr"], t["src"], rev_ptr, rev_perm, dst, r, t["x"], t["w"], t["g"],
                              want=want, frames=frames)
    torch.cuda.synchronize()
    assert etp.device_fault() == 0, "a bounded wait inside a kernel ran out"
    return dict(plan=plan, out=out, rev_ptr=rev_ptr, rev_perm=rev_perm, dst=dst, grad_x=gx, grad_w=gw, grad_r=gr,
                frames=frames)


def compare_full(wl, res, irreps=None):
    irreps = irreps or wl.irreps
    tp = oracle.OracleTP(irreps, wl.L, irreps, wl.C)
    ref_out = tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w)
    ref = tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g)
    errs = {"out": rel_err(res["out"], ref_out)}
    for k in ("grad_x", "grad_w", "grad_r"):
        if res.get(k) is not None:
            errs[k] = rel_err(res[k], ref[k])
    return errs


def compare_sampled(wl, res, n_rows=64, n_nodes=64, n_edges=2048, seed=0):
    """Oracle on a random sample of rows / source nodes / edges (plus first and last)."""
    rng = np.random.default_rng(seed)
    tp = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C)
    rows = np.unique(np.concatenate([[0, wl.N - 1], rng.integers(0, wl.N, n_rows)]))
    nodes = np.unique(np.concatenate([[0, wl.N - 1], rng.integers(0, wl.N, n_nodes)]))
    edges = np.unique(np.concatenate([[0, wl.E - 1], rng.integers(0, wl.E, n_edges)]))
    ref_out = tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, rows=rows)
    ref = tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g, nodes=nodes, edges=edges)
    rows_t, nodes_t, edges_t = (torch.from_numpy(a).to(res["out"].device) for a in (rows, nodes, edges))
    return {
        "out": rel_err(res["out"][rows_t], ref_out),
        "grad_x": rel_err(res["grad_x"][nodes_t], ref["grad_x"]),
        "grad_w": rel_err(res["grad_w"][edges_t], ref["grad_w"]),
        "grad_r": rel_err(res["grad_r"][edges_t], ref["grad_r"]),
    }


def check_errs(errs):
    assert errs["out"] <= FWD_TOL, errs
    for k in ("grad_x", "grad_w", "grad_r"):
        if k in errs:
            assert errs[k] <= VJP_TOL, errs


def check_reverse_csr(wl, res):
    o_rp, o_perm, o_dst = oracle.reverse_csr(wl.N, wl.row_ptr, wl.src)
    assert np.array_equal(res["rev_ptr"].cpu().numpy(), o_rp)
    assert np.array_equal(res["rev_perm"].cpu().numpy(), o_perm)
    if res["dst"] is not None:
        assert np.array_equal(res["dst"].cpu().numpy(), o_dst)


def hub_workload(rng, L, C, P, n=64, hub=20000, rest=3000):
    """A destination with `hub` edges and a source with `hub` edges among n nodes: with
    equal edge ranges per task both hub rows are cut across many tasks."""
    from workloads import Workload, csr_from_pairs

    dst = np.concatenate([np.zeros(hub, np.int64), rng.integers(0, n, hub), rng.integers(0, n, rest)])
    src = np.concatenate([rng.integers(0, n, hub), np.ones(hub, np.int64), rng.integers(0, n, rest)])
    row_ptr, s, _ = csr_from_pairs(n, dst, src)
    E, D = len(s), (L + 1) ** 2
    return Workload("hubs", L, C, P, row_ptr, s, rng.standard_normal((E, 3), dtype=np.float32),
                    rng.standard_normal((n, D, C), dtype=np.float32),
                    rng.standard_normal((E, P, C), dtype=np.float32) / np.float32(np.sqrt(P)),
                    rng.standard_normal((n, D, C), dtype=np.float32))
