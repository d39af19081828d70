"""GPU parity of the fused radial-weights tensor product (etp_fused_forward)
against the FP64 oracle: the radial MLP (oracle.radial.RadialMLP) produces the
per-edge weights in FP64 from the same float32 parameters, and OracleTP sums the
weighted tensor products. Forward tolerance 1e-5 (max error over max |oracle|)."""
import numpy as np
import pytest
import torch

import cg_tensor_products_b200 as etp
import oracle
import workloads
from cg_tensor_products_b200 import build as etp_build
from gpu_helpers import FWD_TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    etp_build.build()
    oracle.build()


def _params(seed, P, C):
    rng = np.random.default_rng(seed)
    W1 = (rng.standard_normal((8, 64)) / np.sqrt(8)).astype(np.float32)
    W2 = (rng.standard_normal((64, P * C)) / np.sqrt(64)).astype(np.float32)
    return W1, W2


def _dev(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


def _oracle_out(irreps, L, C, P, row_ptr, src, r, x, W1, W2, rc, rows=None):
    mlp = oracle.radial.RadialMLP(W1, W2, rc, P, C)
    w = mlp.forward(r)
    return oracle.OracleTP(irreps, L, irreps, C).forward(row_ptr, src, r, x.astype(np.float64), w, rows=rows)


def _fused(plan, row_ptr, src, r, x, W1, W2, rc):
    d = _dev(row_ptr, src, r, x, W1, W2)
    out = etp.fused_forward(plan, *d, rc)
    torch.cuda.synchronize()
    assert etp.device_fault() == 0, "a bounded wait inside a kernel ran out"
    return out, d


@pytest.mark.parametrize("L,o3,C,N,E", [(0, False, 128, 60, 900), (1, False, 8, 40, 700), (1, True, 32, 50, 1500),
                                        (2, False, 64, 70, 3000), (2, True, 16, 30, 1100), (2, False, 4, 20, 333),
                                        (3, False, 128, 90, 2500), (3, True, 64, 64, 1800), (3, False, 8, 17, 515)])
def test_every_spec_ragged_multigraph(L, o3, C, N, E):
    """Ragged random multigraphs (duplicate edges, an empty row, a source without
    edges, a zero-length edge, a ragged last tile) for each slice shape."""
    rng = np.random.default_rng(L * 1000 + C + E)
    P_so3 = workloads.N_PATHS_SO3[L]
    wl = workloads.random_graph(rng, N, E, L, C, P_so3)
    irreps = "+".join(f"{l}{'e' if l % 2 == 0 else 'o'}" for l in range(L + 1)) if o3 else wl.irreps
    plan = etp.Plan(irreps, L, irreps, C)
    P = plan.n_paths
    W1, W2 = _params(L * 7 + C, P, C)
    rc = 5.0
    r = wl.r.copy()
    r[E // 2] = 0.0
    out, _ = _fused(plan, wl.row_ptr, wl.src, r, wl.x, W1, W2, rc)
    ref = _oracle_out(irreps, L, C, P, wl.row_ptr, wl.src, r, wl.x, W1, W2, rc)
    assert rel_err(out, ref) <= FWD_TOL


def test_water_full():
    """The workload whose weights come from the radial MLP, with its own MLP parameters."""
    wl = workloads.make("water")
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    out, d = _fused(plan, wl.row_ptr, wl.src, wl.r, wl.x, wl.W1, wl.W2, wl.r_cut)
    ref = _oracle_out(wl.irreps, wl.L, wl.C, wl.P, wl.row_ptr, wl.src, wl.r, wl.x, wl.W1, wl.W2, wl.r_cut)
    assert rel_err(out, ref) <= FWD_TOL
    # the same result as the unfused chain radial weights -> tensor product
    w = etp.radial_forward(plan, d[2], d[4], d[5], wl.r_cut)
    out2 = etp.forward(plan, d[0], d[1], d[2], d[3], w)
    torch.cuda.synchronize()
    assert rel_err(out, out2.double().cpu().numpy()) <= FWD_TOL


def test_l3_c128_reduced_full():
    """L = 3, C = 128 on a reduced micro graph (200 nodes x 128 neighbours)."""
    wl = workloads.make("micro_l3", n_nodes=200)
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    W1, W2 = _params(33, wl.P, wl.C)
    out, _ = _fused(plan, wl.row_ptr, wl.src, wl.r, wl.x, W1, W2, 6.0)
    ref = _oracle_out(wl.irreps, wl.L, wl.C, wl.P, wl.row_ptr, wl.src, wl.r, wl.x, W1, W2, 6.0)
    assert rel_err(out, ref) <= FWD_TOL


@pytest.mark.parametrize("name", ["micro_l3", "large"])
def test_full_size_sampled_rows(name):
    """Full-size graphs in the benchmark's launch configuration; the oracle evaluates
    sampled rows (first, last and random), from those rows' edges only."""
    wl = workloads.make(name)
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    W1, W2 = _params(44, wl.P, wl.C)
    out, _ = _fused(plan, wl.row_ptr, wl.src, wl.r, wl.x, W1, W2, 6.0)
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, wl.N - 1], rng.integers(0, wl.N, 40)]))
    keep = np.zeros(wl.N, bool)
    keep[rows] = True
    counts = np.diff(wl.row_ptr) * keep
    sub_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    sel = np.repeat(keep, np.diff(wl.row_ptr))
    ref = _oracle_out(wl.irreps, wl.L, wl.C, wl.P, sub_ptr, wl.src[sel], wl.r[sel], wl.x, W1, W2, 6.0, rows=rows)
    assert rel_err(out[torch.from_numpy(rows).cuda()], ref) <= FWD_TOL


def test_repeatable_and_no_edges():
    wl = workloads.make("tiny")
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    W1, W2 = _params(3, wl.P, wl.C)
    a, d = _fused(plan, wl.row_ptr, wl.src, wl.r, wl.x, W1, W2, 5.0)
    b = etp.fused_forward(plan, *d, 5.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    ref = _oracle_out(wl.irreps, wl.L, wl.C, wl.P, wl.row_ptr, wl.src, wl.r, wl.x, W1, W2, 5.0)
    assert rel_err(a, ref) <= FWD_TOL
    # no edges: zeros
    rp = torch.zeros(wl.N + 1, dtype=torch.int32, device="cuda")
    e0 = torch.zeros(0, dtype=torch.int32, device="cuda")
    z = etp.fused_forward(plan, rp, e0, torch.zeros((0, 3), device="cuda"), d[3], d[4], d[5], 5.0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(z) == 0
