"""GPU parity: the CUDA path (through the C ABI) against the FP64 oracle.

Forward <= 1e-5 and VJP <= 1e-4 in max-normalised error per output tensor;
reverse CSR and edge rows bit-exact. Full comparisons at sizes the oracle runs
in seconds (several blocks, ragged tails, empty rows, isolated sources,
duplicate edges); sampled comparisons at the full workload sizes.
"""
import numpy as np
import pytest
import torch

import cg_tensor_products_b200 as etp
import oracle
import oracle.cg
import workloads
from cg_tensor_products_b200 import build as etp_build
from gpu_helpers import (VJP_TOL, check_errs, check_reverse_csr, compare_full, compare_sampled, rel_err, run_gpu,
                         to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    etp_build.build()
    oracle.build()


@pytest.mark.parametrize("framed", [False, True])
@pytest.mark.parametrize("name", ["tiny", "micro_l2", "water"])
def test_workload_full(name, framed):
    wl = workloads.make(name)
    res = run_gpu(wl, framed=framed)
    check_reverse_csr(wl, res)
    errs = compare_full(wl, res)
    print(name, errs)
    check_errs(errs)


@pytest.mark.parametrize("framed", [False, True])
@pytest.mark.parametrize("name", ["micro_l3", "large"])
def test_workload_full_size_sampled(name, framed):
    wl = workloads.make(name)
    res = run_gpu(wl, framed=framed)
    check_reverse_csr(wl, res)
    errs = compare_sampled(wl, res)
    print(name, errs)
    check_errs(errs)
    # invariant at any size: the derivative goes through the direction only
    r = torch.from_numpy(wl.r).cuda().double()
    radial = (res["grad_r"].double() * r).sum(1).abs().max().item()
    scale = (res["grad_r"].double().norm(dim=1) * r.norm(dim=1)).max().item()
    assert radial <= 1e-5 * scale


@pytest.mark.parametrize("framed", [False, True])
def test_l3_c128_reduced_full(framed):
    """The benchmark's shape (L = 3, C = 128, 128 neighbours) on 200 nodes: full comparison."""
    rng = np.random.default_rng(7)
    n, k = 200, 128
    dst = np.repeat(np.arange(n), k)
    src = np.concatenate([np.sort(rng.choice(n, k, replace=False)) for _ in range(n)])
    row_ptr, src_s, order = workloads.csr_from_pairs(n, dst, src)
    E = len(src_s)
    wl = workloads.Workload("l3c128", 3, 128, 34, row_ptr, src_s, (2 * rng.standard_normal((E, 3))).astype(np.float32),
                            rng.standard_normal((n, 16, 128), dtype=np.float32),
                            (rng.standard_normal((E, 34, 128), dtype=np.float32) / np.float32(np.sqrt(34))),
                            rng.standard_normal((n, 16, 128), dtype=np.float32))
    res = run_gpu(wl, framed=framed)
    check_reverse_csr(wl, res)
    errs = compare_full(wl, res)
    print(errs)
    check_errs(errs)


SPECS = [(L, o3, C) for L in range(4) for o3 in (False, True) for C in (4, 8, 16, 32, 64, 128)]


@pytest.mark.parametrize("framed", [False, True])
@pytest.mark.parametrize("L,o3,C", SPECS)
def test_every_compiled_spec_ragged_multigraph(L, o3, C, framed):
    irreps = "+".join(f"{l}{'eo'[l % 2]}" for l in range(L + 1)) if o3 else f"0..{L}"
    P = len(oracle.paths.enumerate_paths(irreps, L, irreps))
    rng = np.random.default_rng(100 * L + C + (7 if o3 else 0))
    wl = workloads.random_graph(rng, 37, 300, L, C, P)
    res = run_gpu(wl, irreps=irreps, with_dst=(C % 8 == 0), framed=framed)  # half: rows by binary search
    check_reverse_csr(wl, res)
    errs = compare_full(wl, res, irreps=irreps)
    check_errs(errs)
    empty = np.flatnonzero(np.diff(wl.row_ptr) == 0)
    assert len(empty) and torch.all(res["out"][torch.from_numpy(empty).cuda()] == 0)
    iso = np.setdiff1d(np.arange(wl.N), wl.src)
    assert len(iso) and torch.all(res["grad_x"][torch.from_numpy(iso).cuda()] == 0)


@pytest.mark.parametrize("want", [("w",), ("r",), ("x",), ("w", "r")])
def test_subsets_of_gradients(want):
    rng = np.random.default_rng(3)
    wl = workloads.random_graph(rng, 50, 400, 2, 32, 15)
    res = run_gpu(wl, want=want)
    full = run_gpu(wl)
    for k, key in (("x", "grad_x"), ("w", "grad_w"), ("r", "grad_r")):
        if k not in want:
            assert res[key] is None
        else:  # node sums included: each output is written once, in a fixed order
            assert torch.equal(res[key], full[key]), key


def test_no_edges():
    n = 9
    wl = workloads.Workload("empty", 2, 16, 15, np.zeros(n + 1, np.int32), np.zeros(0, np.int32),
                            np.zeros((0, 3), np.float32), np.ones((n, 9, 16), np.float32),
                            np.zeros((0, 15, 16), np.float32), np.ones((n, 9, 16), np.float32))
    res = run_gpu(wl)
    assert torch.all(res["out"] == 0) and torch.all(res["grad_x"] == 0)
    assert res["grad_w"].shape == (0, 15, 16) and res["grad_r"].shape == (0, 3)
    assert torch.all(res["rev_ptr"] == 0)


@pytest.mark.parametrize("C", [8, 128])
@pytest.mark.parametrize("framed", [False, True])
def test_zero_length_edge_vectors(framed, C):
    rng = np.random.default_rng(4)
    wl = workloads.random_graph(rng, 20, 120, 3, C, 34)
    wl.r[::7] = 0.0
    res = run_gpu(wl, framed=framed)
    check_errs(compare_full(wl, res))
    assert torch.all(res["grad_r"][::7] == 0)


def test_non_default_stream_and_repeatability():
    """A second run on another stream: every output is bit-identical, node sums
    included (rows cut across several tasks are summed in task order by the
    second pass, without atomics)."""
    wl = workloads.random_graph(np.random.default_rng(5), 64, 2000, 3, 64, 34)
    a = run_gpu(wl)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = run_gpu(wl)
    s.synchronize()
    for k in ("out", "grad_x", "grad_w", "grad_r", "rev_ptr", "rev_perm", "dst"):
        assert torch.equal(a[k], b[k]), k


def test_bitwise_repeatable_when_rows_fit_a_task():
    """Rows no longer than a task (every destination row has 128 edges and the
    tasks are 128 edges long): every output repeats bit for bit."""
    rng = np.random.default_rng(9)
    n, k = 300, 128
    dst = np.repeat(np.arange(n), k)
    src = np.concatenate([np.sort(rng.choice(n, k, replace=False)) for _ in range(n)])
    row_ptr, src_s, _ = workloads.csr_from_pairs(n, dst, src)
    E = len(src_s)
    wl = workloads.Workload("rep", 2, 128, 15, row_ptr, src_s, rng.standard_normal((E, 3), dtype=np.float32),
                            rng.standard_normal((n, 9, 128), dtype=np.float32),
                            rng.standard_normal((E, 15, 128), dtype=np.float32),
                            rng.standard_normal((n, 9, 128), dtype=np.float32))
    a, b = run_gpu(wl), run_gpu(wl)
    for key in ("out", "grad_x", "grad_w", "grad_r"):
        assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("n,e", [(1, 0), (1, 50), (2, 7), (256, 5000), (257, 5000), (70000, 300000),
                                 (3, 10000), (2048, 200000), (2049, 200000), (1024, 131072),
                                 (1500, 2_200_000), (3072, 166518), (8192, 300000), (8193, 300000),
                                 (4000, 1_000_000), (4000, 1_100_000)])
def test_reverse_csr_bit_exact(n, e):
    rng = np.random.default_rng(n + e)
    dst = rng.integers(0, n, e)
    src = rng.integers(0, n, e)
    row_ptr, s, _ = workloads.csr_from_pairs(n, dst, src)
    rp, perm, d = etp.build_reverse_csr(n, torch.from_numpy(row_ptr).cuda(), torch.from_numpy(s).cuda())
    o_rp, o_perm, o_d = oracle.reverse_csr(n, row_ptr, s)
    assert np.array_equal(rp.cpu().numpy(), o_rp)
    assert np.array_equal(perm.cpu().numpy(), o_perm)
    assert np.array_equal(d.cpu().numpy(), o_d)


def test_validate_csr_flags():
    dev = "cuda:0"
    rp = torch.tensor([0, 2, 3, 5], dtype=torch.int32, device=dev)
    src = torch.tensor([1, 2, 0, 0, 1], dtype=torch.int32, device=dev)
    assert etp.validate_csr(3, rp, src) == 0
    assert etp.validate_csr(3, torch.tensor([1, 2, 3, 5], dtype=torch.int32, device=dev), src) & etp.CSR_BAD_ENDPOINTS
    assert etp.validate_csr(3, torch.tensor([0, 2, 3, 4], dtype=torch.int32, device=dev), src) & etp.CSR_BAD_ENDPOINTS
    assert etp.validate_csr(3, torch.tensor([0, 3, 2, 5], dtype=torch.int32, device=dev), src) == etp.CSR_NOT_MONOTONE
    assert etp.validate_csr(3, rp, torch.tensor([1, 2, 3, 0, 1], dtype=torch.int32, device=dev)) == etp.CSR_SRC_RANGE
    assert etp.validate_csr(3, rp, torch.tensor([1, -1, 0, 0, 1], dtype=torch.int32, device=dev)) == etp.CSR_SRC_RANGE


def test_out_of_range_sources_are_skipped_not_faulted():
    """An invalid src (caught by validate_csr) must not make the kernels leave their buffers;
    such edges contribute nothing, and their grad_w and grad_r are zero."""
    rng = np.random.default_rng(6)
    wl = workloads.random_graph(rng, 16, 100, 1, 8, 5)
    t = to_dev(wl)
    bad_src = t["src"].clone()
    bad_src[::9] = 1 << 20
    plan = etp.Plan("0..1", 1, "0..1", 8)
    assert etp.validate_csr(wl.N, t["row_ptr"], bad_src) == etp.CSR_SRC_RANGE
    out = etp.forward(plan, t["row_ptr"], bad_src, t["r"], t["x"], t["w"])
    torch.cuda.synchronize()
    keep = np.ones(wl.E, bool)
    keep[::9] = False
    # the same graph with those edges given zero weight is the reference
    w0 = wl.w.copy()
    w0[~keep] = 0
    tp = oracle.OracleTP("0..1", 1, "0..1", 8)
    ref = tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, w0)
    assert rel_err(out, ref) <= 1e-5
    # the VJP: those edges add nothing to grad_x and get zero grad_w and grad_r
    rev_ptr, rev_perm, dst = etp.build_reverse_csr(wl.N, t["row_ptr"], bad_src)
    gx, gw, gr = etp.backward(plan, t["row_ptr"], bad_src, rev_ptr, rev_perm, dst, t["r"], t["x"], t["w"], t["g"])
    torch.cuda.synchronize()
    assert etp.device_fault() == 0
    ref_b = tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, w0, wl.g)
    bad = torch.from_numpy(~keep).cuda()
    assert torch.count_nonzero(gw[bad]) == 0 and torch.count_nonzero(gr[bad]) == 0
    assert rel_err(gx, ref_b["grad_x"]) <= 1e-4
    assert rel_err(gw[~bad], ref_b["grad_w"][keep]) <= 1e-4
    assert rel_err(gr[~bad], ref_b["grad_r"][keep]) <= 1e-4


@pytest.mark.parametrize("L", [0, 1, 2, 3])
def test_edge_frame_records(L):
    """The frame record of each edge: R a proper rotation taking r/|r| to z,
    1/|r|, the zero-length flag, and D_2, D_3 equal to the oracle's Wigner
    matrices of that R (Y_l(R u) = D_l(R) Y_l(u))."""
    rng = np.random.default_rng(11 + L)
    E = 300
    r = rng.standard_normal((E, 3)).astype(np.float32) * rng.uniform(0.1, 5.0, (E, 1)).astype(np.float32)
    r[5] = 0.0
    r[17] = (1e-14, 0.0, 0.0)
    r[30] = (0.0, 0.0, -2.5)   # on the axis opposite z
    r[31] = (0.0, 0.0, 3.0)
    plan = etp.Plan(f"0..{L}", L, f"0..{L}", 8)
    fr = etp.edge_frames(plan, torch.from_numpy(r).cuda())
    torch.cuda.synchronize()
    fr = fr.cpu().numpy().astype(np.float64)
    assert fr.shape == (E, etp.FRAME_FLOATS)
    n = np.linalg.norm(r.astype(np.float64), axis=1)
    for e in range(E):
        R = fr[e, 76:85].reshape(3, 3)
        if n[e] < 1e-12:
            assert fr[e, 86] == 1.0 and fr[e, 85] == 0.0
            assert np.allclose(R, np.eye(3))
            continue
        assert fr[e, 86] == 0.0
        assert abs(fr[e, 85] * n[e] - 1) < 1e-6
        assert np.abs(R @ R.T - np.eye(3)).max() < 1e-6 and abs(np.linalg.det(R) - 1) < 1e-6
        assert np.abs(R @ (r[e] / n[e]) - np.array([0.0, 0.0, 1.0])).max() < 1e-6
        if L >= 2:
            assert np.abs(fr[e, 0:25].reshape(5, 5) - oracle.cg.wigner_d(2, R)).max() < 2e-5, e
        if L >= 3:
            assert np.abs(fr[e, 25:74].reshape(7, 7) - oracle.cg.wigner_d(3, R)).max() < 2e-5, e


def test_framed_and_unframed_agree():
    """Both kernel variants evaluate the same frames: results agree to rounding."""
    wl = workloads.random_graph(np.random.default_rng(12), 80, 3000, 3, 128, 34)
    a, b = run_gpu(wl), run_gpu(wl, framed=True)
    for k in ("out", "grad_x", "grad_w", "grad_r"):
        assert rel_err(a[k], b[k].double().cpu().numpy()) <= 1e-6, k


@pytest.mark.parametrize("n", [100, 5000])
def test_reverse_csr_with_out_of_range_sources(n):
    """Sources outside [0, N) (an invalid CSR) are grouped after all valid ones:
    rev_ptr[N] counts the valid edges, the valid part matches the stable grouping
    of the valid edges, and rev_perm stays a permutation (nothing out of bounds)."""
    rng = np.random.default_rng(n)
    e = 20000
    dst = rng.integers(0, n, e)
    src = rng.integers(0, n, e)
    row_ptr, s, _ = workloads.csr_from_pairs(n, dst, src)
    s = s.copy()
    bad = rng.random(e) < 0.05
    s[bad] = np.where(rng.random(bad.sum()) < 0.5, -3, n + 7)
    rp, perm, d = etp.build_reverse_csr(n, torch.from_numpy(row_ptr).cuda(), torch.from_numpy(s).cuda())
    rp, perm = rp.cpu().numpy(), perm.cpu().numpy()
    valid = np.flatnonzero(~bad)
    order = valid[np.argsort(s[valid], kind="stable")]
    assert rp[n] == len(valid)
    assert np.array_equal(perm[:len(valid)], order)
    assert np.array_equal(np.sort(perm), np.arange(e))
    assert np.array_equal(rp, np.concatenate([[0], np.cumsum(np.bincount(s[valid], minlength=n))]))


@pytest.mark.parametrize("framed", [False, True])
def test_hub_rows_cut_across_many_tasks(framed):
    """A destination with 20,000 edges and a source with 20,000 edges among 64 nodes:
    the tasks are equal edge ranges, so both hub rows are cut across ~30 tasks and
    their pieces are summed in task order by the second pass: results compare with
    the oracle and repeat bit for bit."""
    rng = np.random.default_rng(21)
    n, hub = 64, 20000
    dst = np.concatenate([np.zeros(hub, np.int64), rng.integers(0, n, hub), rng.integers(0, n, 3000)])
    src = np.concatenate([rng.integers(0, n, hub), np.ones(hub, np.int64), rng.integers(0, n, 3000)])
    row_ptr, s, _ = workloads.csr_from_pairs(n, dst, src)
    E = len(s)
    wl = workloads.Workload("hubs", 3, 32, 34, row_ptr, s, rng.standard_normal((E, 3), dtype=np.float32),
                            rng.standard_normal((n, 16, 32), dtype=np.float32),
                            rng.standard_normal((E, 34, 32), dtype=np.float32) / np.float32(np.sqrt(34)),
                            rng.standard_normal((n, 16, 32), dtype=np.float32))
    res = run_gpu(wl, framed=framed)
    check_reverse_csr(wl, res)
    errs = compare_full(wl, res)
    print(errs)
    check_errs(errs)
    again = run_gpu(wl, framed=framed)
    for k in ("out", "grad_x", "grad_w", "grad_r"):
        assert torch.equal(res[k], again[k]), k


@pytest.mark.parametrize("name", ["tiny", "water", "micro_l3"])
def test_assembled_forces_match_oracle(name):
    """Forces and per-atom virials from the GPU's grad_r against the oracle's
    assembly of the oracle's grad_r (VJP tolerance), momentum conservation, and
    bit-for-bit repetition."""
    wl = workloads.make(name)
    res = run_gpu(wl, framed=True)
    r = torch.from_numpy(wl.r).cuda()
    rp = torch.from_numpy(wl.row_ptr).cuda()
    F, V = etp.assemble_forces(wl.N, rp, res["rev_ptr"], res["rev_perm"], res["grad_r"], r=r)
    F2, V2 = etp.assemble_forces(wl.N, rp, res["rev_ptr"], res["rev_perm"], res["grad_r"], r=r)
    F3, V3 = etp.assemble_forces(wl.N, rp, res["rev_ptr"], res["rev_perm"], res["grad_r"])
    torch.cuda.synchronize()
    assert torch.equal(F, F2) and torch.equal(V, V2) and torch.equal(F, F3) and V3 is None
    tp = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C)
    if name == "micro_l3":   # grad_r of a sample of edges is enough to pin the oracle side here
        edges = np.arange(wl.E)
        g_ref = np.concatenate([tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g, nodes=np.arange(1),
                                            edges=edges[k:k + 32768], want=("r",))["grad_r"]
                                for k in range(0, wl.E, 32768)])
    else:
        g_ref = tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g, want=("r",))["grad_r"]
    F_ref, V_ref = oracle.assemble_forces(wl.N, wl.row_ptr, wl.src, wl.r, g_ref)
    assert rel_err(F, F_ref) <= VJP_TOL and rel_err(V, V_ref) <= VJP_TOL
    # the GPU assembly itself, on the GPU's own grad_r, to fp32 summation accuracy
    F_own, V_own = oracle.assemble_forces(wl.N, wl.row_ptr, wl.src, wl.r, res["grad_r"].double().cpu().numpy())
    assert rel_err(F, F_own) <= 1e-5 and rel_err(V, V_own) <= 1e-5
    assert F.double().sum(0).abs().max().item() <= 1e-5 * res["grad_r"].double().abs().sum().item()


def test_cuda_graph_capture_and_replay():
    """The whole step (reverse CSR, frames, forward, VJP, forces) captured once into a
    CUDA graph and replayed on new input values gives what eager calls give."""
    rng = np.random.default_rng(31)
    wl = workloads.random_graph(rng, 300, 9000, 3, 64, 34)
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    t = to_dev(wl)
    N, E = wl.N, wl.E
    outs = dict(out=torch.empty(N, 16, 64, device="cuda"), gx=torch.empty(N, 16, 64, device="cuda"),
                gw=torch.empty(E, 34, 64, device="cuda"), gr=torch.empty(E, 3, device="cuda"),
                frames=torch.empty(E, etp.FRAME_FLOATS, device="cuda"), F=torch.empty(N, 3, device="cuda"),
                ws=torch.empty(etp.reverse_csr_workspace_size(N, E), dtype=torch.uint8, device="cuda"))

    def step():
        rp, perm, dst = etp.build_reverse_csr(N, t["row_ptr"], t["src"], workspace=outs["ws"])
        etp.edge_frames(plan, t["r"], frames=outs["frames"])
        etp.forward(plan, t["row_ptr"], t["src"], None, t["x"], t["w"], out=outs["out"], frames=outs["frames"])
        etp.backward(plan, t["row_ptr"], t["src"], rp, perm, dst, None, t["x"], t["w"], t["g"], grad_x=outs["gx"],
                     grad_w=outs["gw"], grad_r=outs["gr"], frames=outs["frames"])
        etp.assemble_forces(N, t["row_ptr"], rp, perm, outs["gr"], forces=outs["F"])

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                        # warm-up outside capture (fills the launch-shape caches)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for trial in range(2):
        for k in ("r", "x", "w", "g"):
            t[k].copy_(torch.randn_like(t[k]))
        graph.replay()
        torch.cuda.synchronize()
        got = {k: outs[k].clone() for k in ("out", "gx", "gw", "gr", "F")}
        step()
        torch.cuda.synchronize()
        assert etp.device_fault() == 0
        for k, v in got.items():
            assert rel_err(v, outs[k].double().cpu().numpy()) <= 1e-6, (trial, k)
