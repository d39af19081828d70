"""GPU parity of the Cartesian edge convolution (etp_cart_forward / etp_cart_backward)
against the FP64 Cartesian oracle (oracle/cartesian.py, full 3^l tensors, VJP by
autograd). The library holds a rank-l STF tensor by its 2l + 1 entries with at most
one z index; the test maps those to and from full tensors with its own expansion
(STF completion) and entry picks. Tolerances: forward 1e-5, VJP 1e-4."""

import numpy as np
import pytest
import torch

import cg_tensor_products_b200 as etp
import oracle
import workloads
from cg_tensor_products_b200 import build as etp_build
from gpu_helpers import FWD_TOL, VJP_TOL, rel_err
from cart_layout import expand as _expand, from_full as _from_full, pick as _pick, to_full as _to_full
from oracle import cartesian as ct

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    etp_build.build()
    oracle.build()


def _run(wl, irreps, w, r):
    plan = etp.Plan(irreps, wl.L, irreps, wl.C)
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    rp, src = dv(wl.row_ptr), dv(wl.src)
    out = etp.cart_forward(plan, rp, src, dv(r), dv(wl.x), dv(w))
    rev_ptr, rev_perm, dst = etp.build_reverse_csr(wl.N, rp, src)
    gx, gw, gr = etp.cart_backward(plan, rp, src, rev_ptr, rev_perm, dst, dv(r), dv(wl.x), dv(w), dv(wl.g))
    torch.cuda.synchronize()
    assert etp.device_fault() == 0
    return out, gx, gw, gr


def _oracle(wl, irreps, w, r, row_ptr=None, src=None):
    row_ptr = wl.row_ptr if row_ptr is None else row_ptr
    src = wl.src if src is None else src
    tp = ct.OracleCartTP(irreps, wl.L, irreps, wl.C)
    xf = _to_full(wl.x, wl.L)
    out = tp.forward(row_ptr, src, r, xf, w)
    out_c = _from_full(out, wl.L, _pick)
    # the loss <out, g> over independent components is <out_full, S^T g>
    g_full = {l: torch.from_numpy(np.einsum("if,nic->ncf", _pick(l), wl.g[:, l * l:(l + 1) ** 2, :].astype(np.float64))
                                  .reshape(wl.N, wl.C, *([3] * l)) if l else
                                  wl.g[:, 0, :].astype(np.float64)) for l in range(wl.L + 1)}
    b = tp.backward(row_ptr, src, r, xf, w, g_full)
    gx_c = _from_full(b["grad_x"], wl.L, lambda l: _expand(l).T)    # chain rule through x_full = E x
    # with harmonics of degree 0 only, r does not enter the output: its gradient is zero
    gr = b["grad_r"].numpy() if b["grad_r"] is not None else np.zeros((len(src), 3))
    return out_c, gx_c, b["grad_w"].numpy(), gr


@pytest.mark.parametrize("L,o3,C,N,E", [(0, False, 8, 20, 300), (1, False, 8, 40, 700), (1, True, 32, 30, 900),
                                        (2, False, 64, 50, 1500), (2, True, 16, 30, 800), (2, False, 4, 17, 333),
                                        (3, False, 128, 40, 1200), (3, True, 64, 33, 1000), (3, False, 8, 20, 515)])
def test_every_spec_ragged_multigraph(L, o3, C, N, E):
    """Every compiled specialisation on a ragged random multigraph with an empty row,
    a source without edges and a zero-length edge."""
    rng = np.random.default_rng(L * 31 + C + E)
    wl = workloads.random_graph(rng, N, E, L, C, workloads.N_PATHS_SO3[L])
    irreps = "+".join(f"{l}{'e' if l % 2 == 0 else 'o'}" for l in range(L + 1)) if o3 else wl.irreps
    P = etp.Plan(irreps, L, irreps, C).n_paths
    w = (rng.standard_normal((E, P, C)) / np.sqrt(P)).astype(np.float32)
    r = wl.r.copy()
    r[E // 4] = 0.0
    out, gx, gw, gr = _run(wl, irreps, w, r)
    ref = _oracle(wl, irreps, w, r)
    assert rel_err(out, ref[0]) <= FWD_TOL
    assert rel_err(gx, ref[1]) <= VJP_TOL
    assert rel_err(gw, ref[2]) <= VJP_TOL
    assert rel_err(gr, ref[3]) <= VJP_TOL


@pytest.mark.parametrize("name", ["micro_l2", "micro_l3"])
def test_micro_sampled_rows(name):
    """The micro-benchmark graphs at full size (the comparison with the spherical
    kernel at equal rank); the oracle runs on sampled rows' edges."""
    wl = workloads.make(name)
    out, gx, gw, gr = _run(wl, wl.irreps, wl.w, wl.r)
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, wl.N - 1], rng.integers(0, wl.N, 6)]))
    keep = np.repeat(np.isin(np.arange(wl.N), rows), np.diff(wl.row_ptr))
    counts = np.diff(wl.row_ptr) * np.isin(np.arange(wl.N), rows)
    sub_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    sub = workloads.Workload(wl.name, wl.L, wl.C, wl.P, sub_ptr, wl.src[keep], wl.r[keep], wl.x, wl.w[keep], wl.g)
    ref = _oracle(sub, wl.irreps, wl.w[keep], wl.r[keep])
    sel = torch.from_numpy(rows).cuda()
    assert rel_err(out[sel], ref[0][rows]) <= FWD_TOL
    idx = torch.from_numpy(np.nonzero(keep)[0]).cuda()
    assert rel_err(gw[idx], ref[2]) <= VJP_TOL
    assert rel_err(gr[idx], ref[3]) <= VJP_TOL


@pytest.mark.parametrize("C", [16, 128])
def test_hub_rows_repeatable(C):
    """Hub rows cut across many tasks: oracle parity, and two runs agree bit for bit."""
    from gpu_helpers import hub_workload

    wl = hub_workload(np.random.default_rng(37), 2, C, 15, hub=6000, rest=1000)
    a = _run(wl, wl.irreps, wl.w, wl.r)
    b = _run(wl, wl.irreps, wl.w, wl.r)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    ref = _oracle(wl, wl.irreps, wl.w, wl.r)
    assert rel_err(a[0], ref[0]) <= FWD_TOL
    assert rel_err(a[1], ref[1]) <= VJP_TOL
    assert rel_err(a[2], ref[2]) <= VJP_TOL
    assert rel_err(a[3], ref[3]) <= VJP_TOL
