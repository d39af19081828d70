"""GPU checks of the locality schedule (etp_build_locality_schedule,
etp_forward_ordered, etp_backward_ordered).

The schedule is index work: it is compared bit for bit with a host restatement of
its definition (bounding box, cells of side max(cell, extent / 1023), Morton code
with 10 bits per axis, stable sort; rows and sources taken in that order). The
ordered kernels compute the same sums as the unordered ones, so they are compared
with the FP64 oracle at the usual tolerances (forward 1e-5, VJP 1e-4), and with the
unordered kernels at 1e-6: only the rows cut by a task boundary, which differ
between the two schedules, are summed in another order.
"""
import numpy as np
import pytest
import torch

import cg_tensor_products_b200 as etp
import oracle
import workloads
from cg_tensor_products_b200 import build as etp_build
from gpu_helpers import check_errs, compare_full, compare_sampled, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    etp_build.build()
    oracle.build()


def _spread3(v):
    v = v.astype(np.uint64) & 0x3FF
    out = np.zeros_like(v)
    for b in range(10):
        out |= ((v >> b) & 1) << (3 * b)
    return out


def host_order(pos, cell):
    """The schedule's node order, restated in float32 on the host."""
    p = pos.astype(np.float32)
    nan = np.isnan(p)
    lo = np.where(nan, np.float32(np.inf), p).min(0)
    hi = np.where(nan, np.float32(-np.inf), p).max(0)
    ext = np.float32(max(hi[0] - lo[0], hi[1] - lo[1], hi[2] - lo[2]))
    side = np.float32(max(np.float32(cell), np.float32(ext * (np.float32(1.0) / np.float32(1023.0)))))
    inv = np.float32(1.0) / side
    with np.errstate(invalid="ignore"):
        t = ((p - lo) * inv).astype(np.float32)
        c = np.where(t >= 1023, 1023, np.where(t > 0, np.floor(np.nan_to_num(t)), 0)).astype(np.uint64)
    key = _spread3(c[:, 0]) | (_spread3(c[:, 1]) << 1) | (_spread3(c[:, 2]) << 2)
    return np.argsort(key, kind="stable").astype(np.int32)


def host_schedule(row_ptr, src, order):
    N = len(row_ptr) - 1
    rank = np.empty(N, dtype=np.int64)
    rank[order] = np.arange(N)
    deg = np.diff(row_ptr)[order]
    ord_ptr = np.concatenate([[0], np.cumsum(deg)]).astype(np.int32)
    ord_edge = np.concatenate([np.arange(row_ptr[i], row_ptr[i + 1]) for i in order] or [[]]).astype(np.int32)
    keys = rank[src]
    rev_perm = np.argsort(keys, kind="stable").astype(np.int32)
    rev_ptr = np.concatenate([[0], np.cumsum(np.bincount(keys, minlength=N))]).astype(np.int32)
    dst = np.repeat(np.arange(N), np.diff(row_ptr)).astype(np.int32)
    return ord_ptr, ord_edge, rev_ptr, rev_perm, dst


def _random_pos(rng, N, box=20.0):
    return rng.uniform(0.0, box, size=(N, 3)).astype(np.float32)


def _schedule(wl, pos, cell):
    t = to_dev(wl)
    s = etp.locality_schedule(wl.N, t["row_ptr"], t["src"], torch.from_numpy(pos).cuda(), cell)
    torch.cuda.synchronize()
    return t, s


def _check_schedule(wl, pos, cell, s):
    order = host_order(pos, cell)
    assert np.array_equal(s.order.cpu().numpy(), order)
    want = host_schedule(wl.row_ptr, wl.src, order)
    for got, ref in zip((s.ord_ptr, s.ord_edge, s.rev_ptr, s.rev_perm, s.dst), want):
        assert np.array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("name", ["tiny", "water", "large"])
def test_schedule_bit_exact(name):
    wl = workloads.make(name)
    pos = wl.pos if wl.pos is not None else _random_pos(np.random.default_rng(1), wl.N)
    cell = wl.graph_cutoff or 2.0
    _, s = _schedule(wl, pos, cell)
    _check_schedule(wl, pos, cell, s)


@pytest.mark.parametrize("N,E", [(1, 0), (1, 5), (17, 333), (300, 9000), (9000, 70000)])
def test_schedule_edge_cases(N, E):
    """One node, no edges, empty rows, sources without edges, coincident and NaN
    positions, a cell larger than the box and one far smaller (extent / 1023 wins)."""
    rng = np.random.default_rng(N + E)
    wl = workloads.random_graph(rng, N, E, 1, 8, 5)
    pos = _random_pos(rng, N)
    if N > 4:
        pos[3] = pos[2]
        pos[4, 1] = np.nan
    for cell in (0.5, 1e-6, 1e6):
        _, s = _schedule(wl, pos, cell)
        _check_schedule(wl, pos, cell, s)


def _run_ordered(wl, plan, t, s, framed):
    frames = etp.edge_frames(plan, t["r"]) if framed else None
    r = None if framed else t["r"]
    out = etp.forward_ordered(plan, s, t["src"], r, t["x"], t["w"], frames=frames)
    gx, gw, gr = etp.backward_ordered(plan, s, r, t["x"], t["w"], t["g"], frames=frames)
    torch.cuda.synchronize()
    assert etp.device_fault() == 0
    return dict(out=out, grad_x=gx, grad_w=gw, grad_r=gr)


def _run_plain(wl, plan, t):
    out = etp.forward(plan, t["row_ptr"], t["src"], t["r"], t["x"], t["w"])
    rev_ptr, rev_perm, dst = etp.build_reverse_csr(wl.N, t["row_ptr"], t["src"])
    gx, gw, gr = etp.backward(plan, t["row_ptr"], t["src"], rev_ptr, rev_perm, dst, t["r"], t["x"], t["w"], t["g"])
    torch.cuda.synchronize()
    return dict(out=out, grad_x=gx, grad_w=gw, grad_r=gr)


def _agree(a, b, tol=1e-6):
    for k in ("out", "grad_x", "grad_w", "grad_r"):
        ref = b[k].double().cpu().numpy()
        assert rel_err(a[k], ref) <= tol, k


@pytest.mark.parametrize("framed", [False, True])
def test_ordered_water_full(framed):
    wl = workloads.make("water")
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    t, s = _schedule(wl, wl.pos, wl.graph_cutoff)
    res = _run_ordered(wl, plan, t, s, framed)
    check_errs(compare_full(wl, res))
    _agree(res, _run_plain(wl, plan, t))


@pytest.mark.parametrize("framed", [False, True])
def test_ordered_large_sampled(framed):
    wl = workloads.make("large")
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    t, s = _schedule(wl, wl.pos, wl.graph_cutoff)
    res = _run_ordered(wl, plan, t, s, framed)
    check_errs(compare_sampled(wl, res))
    _agree(res, _run_plain(wl, plan, t))


SPECS = [(0, False, 8), (1, True, 32), (2, False, 64), (2, True, 16), (3, False, 128), (3, True, 64), (3, False, 4)]


@pytest.mark.parametrize("L,o3,C", SPECS)
def test_ordered_every_spec_ragged(L, o3, C):
    rng = np.random.default_rng(L * 7 + C)
    wl = workloads.random_graph(rng, 41, 1500, L, C, workloads.N_PATHS_SO3[L])
    irreps = "+".join(f"{l}{'e' if l % 2 == 0 else 'o'}" for l in range(L + 1)) if o3 else wl.irreps
    plan = etp.Plan(irreps, L, irreps, C)
    wl.w = (rng.standard_normal((wl.E, plan.n_paths, C)) / np.sqrt(plan.n_paths)).astype(np.float32)
    wl.r[7] = 0.0
    t, s = _schedule(wl, _random_pos(rng, wl.N), 3.0)
    res = _run_ordered(wl, plan, t, s, False)
    check_errs(compare_full(wl, res, irreps=irreps))


def test_ordered_bitwise_repeatable():
    """Two schedules of the same graph and two runs on them: every output repeats bit for bit."""
    wl = workloads.make("water")
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    t, s = _schedule(wl, wl.pos, wl.graph_cutoff)
    a = _run_ordered(wl, plan, t, s, False)
    _, s2 = _schedule(wl, wl.pos, wl.graph_cutoff)
    b = _run_ordered(wl, plan, t, s2, False)
    for k in a:
        assert torch.equal(a[k], b[k]), k
