"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
declared symbol, builds plans whose paths and compiled couplings agree with the
oracle's independent construction, and rejects bad arguments before any launch.

Every call below that passes pointers is built to fail a host check (a NULL, a
negative size or a misaligned address), so no kernel is ever launched here.
"""
import ctypes

import numpy as np
import pytest

import cg_tensor_products_b200 as etp
from cg_tensor_products_b200 import build as etp_build
from oracle import cg, paths


@pytest.fixture(scope="module")
def lib():
    etp_build.build()
    return etp._load()


def test_exports_every_declared_symbol(lib):
    names = etp.declared_symbols()
    assert len(names) == 30
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("L,o3", [(L, o3) for L in range(4) for o3 in (False, True)])
def test_plan_paths_match_oracle(lib, L, o3):
    irreps = "+".join(f"{l}{'eo'[l % 2]}" for l in range(L + 1)) if o3 else f"0..{L}"
    plan = etp.Plan(irreps, L, irreps, 64)
    assert plan.paths == paths.enumerate_paths(irreps, L, irreps)
    assert plan.dim_in == plan.dim_out == (L + 1) ** 2


@pytest.mark.parametrize("L", [1, 2, 3])
def test_compiled_couplings_match_oracle_construction(lib, L):
    """Racah-formula tables (library) vs invariance construction (oracle): 1e-12."""
    plan = etp.Plan(f"0..{L}", L, f"0..{L}", 8)
    off, m1, m2, m3, val = plan.couplings()
    for p, (l1, l2, l3) in enumerate(plan.paths):
        T = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
        for k in range(off[p], off[p + 1]):
            T[m1[k], m2[k], m3[k]] = val[k]
        assert np.max(np.abs(T - cg.real_cg(l1, l2, l3))) < 1e-12, (l1, l2, l3)
        assert off[p + 1] - off[p] == len(cg.nnz_list(l1, l2, l3))


def _create(lib, a, lmax, b, C, dtype=0):
    h = ctypes.c_void_p()
    st = lib.etp_plan_create(ctypes.byref(h), a.encode(), lmax, b.encode(), C, dtype)
    if st == 0:
        lib.etp_plan_destroy(h)
    return st


def test_plan_create_rejections(lib):
    assert _create(lib, "0..3", 3, "0..3", 128) == etp.ETP_OK
    assert _create(lib, "0+1+2", 2, "0+1+2", 64) == etp.ETP_OK
    assert _create(lib, "0e+1o+2e+3o", 3, "0e+1o+2e+3o", 8) == etp.ETP_OK
    for C in (4, 8, 16, 32, 64, 128):
        assert _create(lib, "0..1", 1, "0..1", C) == etp.ETP_OK
    unsupported = [("0..4", 4, "0..4", 8), ("0..2", 3, "0..2", 8), ("0..2", 2, "0..1", 8), ("1..2", 2, "1..2", 8),
                   ("0..2", 2, "0..2", 12), ("0..2", 2, "0..2", 256), ("0..2", 2, "0..2", 6),
                   ("0o+1e", 1, "0o+1e", 8), ("0+2", 2, "0+2", 8)]
    for args in unsupported:
        assert _create(lib, *args) == etp.ETP_ERR_UNSUPPORTED, args
    assert _create(lib, "0..2", 2, "0..2", 8, dtype=3) == etp.ETP_ERR_UNSUPPORTED
    invalid = [("", 1, "0..1", 8), ("0+x", 1, "0..1", 8), ("0++1", 1, "0..1", 8), ("1+0", 1, "1+0", 8),
               ("0e+1", 1, "0e+1", 8), ("0e+1o", 1, "0+1", 8), ("0..1", -1, "0..1", 8), ("0..1", 1, "0..1", 0),
               ("3..1", 1, "0..1", 8)]
    for args in invalid:
        assert _create(lib, *args) == etp.ETP_ERR_INVALID_ARG, args
    assert lib.etp_plan_create(None, b"0..1", 1, b"0..1", 8, 0) == etp.ETP_ERR_INVALID_ARG


def test_host_argument_checks(lib):
    h = ctypes.c_void_p()
    assert lib.etp_plan_create(ctypes.byref(h), b"0..2", 2, b"0..2", 64, 0) == 0
    ok = ctypes.c_void_p(0x10000)       # never dereferenced: each call fails a host check
    bad = ctypes.c_void_p(0x10004)      # not 16-byte aligned
    F = lib.etp_forward
    assert F(None, 4, 4, ok, ok, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG       # no plan
    assert F(h, -1, 4, ok, ok, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG         # N < 0
    assert F(h, 4, -2, ok, ok, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG         # E < 0
    assert F(h, 0, 3, ok, ok, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG          # edges without nodes
    assert F(h, 0, 0, None, None, None, None, None, None, None, ok, 1 << 30, None) == etp.ETP_OK           # nothing to do
    assert F(h, 4, 4, None, ok, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG        # row_ptr NULL
    assert F(h, 4, 4, ok, ok, ok, None, bad, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG         # x misaligned
    assert F(h, 4, 4, ok, ok, ok, None, ok, bad, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG         # w misaligned
    assert F(h, 4, 4, ok, ok, ok, None, ok, ok, bad, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG         # out misaligned
    assert F(h, 4, 4, ok, None, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG        # src NULL with E > 0
    assert F(h, 4, 4, ok, ok, None, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG     # neither r nor frames
    assert F(h, 4, 4, ok, ok, None, bad, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG      # frames misaligned
    assert F(h, 4, 4, ok, ok, ok, None, ok, ok, ok, None, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG  # no workspace
    assert F(h, 4, 4, ok, ok, ok, None, ok, ok, ok, bad, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG   # misaligned
    assert F(h, 4, 4, ok, ok, ok, None, ok, ok, ok, ok, 0, None) == etp.ETP_ERR_WORKSPACE             # too small
    B = lib.etp_backward
    assert B(h, 4, 4, ok, ok, None, ok, ok, ok, None, ok, ok, ok, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG  # rev_ptr
    assert B(h, 4, 4, ok, ok, ok, None, ok, ok, None, ok, ok, ok, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG  # rev_perm
    assert B(h, 4, 4, ok, ok, ok, ok, ok, ok, None, ok, ok, bad, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG   # grad_out
    assert B(h, 4, 4, ok, ok, ok, ok, ok, ok, None, ok, ok, ok, ok, bad, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG   # grad_w
    assert B(h, 4, 4, ok, ok, ok, ok, ok, ok, None, ok, ok, ok, bad, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG   # grad_x
    assert B(h, 4, 4, ok, ok, ok, ok, ok, ok, None, ok, ok, ok, None, None, None, ok, 1 << 30, None) == etp.ETP_OK  # nothing wanted
    assert B(h, 4, 4, ok, ok, ok, ok, ok, None, None, ok, ok, ok, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG  # no r/frames
    assert B(h, 4, 4, ok, ok, ok, ok, ok, None, bad, ok, ok, ok, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG   # frames
    assert B(h, 4, 4, ok, ok, ok, ok, ok, ok, None, ok, ok, ok, ok, ok, ok, ok, 0, None) == etp.ETP_ERR_WORKSPACE
    tw = ctypes.c_size_t()
    assert lib.etp_tp_workspace_size(h, 100, 1000, 0, ctypes.byref(tw)) == etp.ETP_OK and tw.value > 0
    assert lib.etp_tp_workspace_size(h, 100, 0, 0, ctypes.byref(tw)) == etp.ETP_OK and tw.value == 0
    assert lib.etp_tp_workspace_size(None, 100, 1000, 0, ctypes.byref(tw)) == etp.ETP_ERR_INVALID_ARG
    G = lib.etp_edge_frames
    assert G(None, 4, ok, ok, None) == etp.ETP_ERR_INVALID_ARG      # no plan
    assert G(h, -1, ok, ok, None) == etp.ETP_ERR_INVALID_ARG        # E < 0
    assert G(h, 4, None, ok, None) == etp.ETP_ERR_INVALID_ARG       # r NULL
    assert G(h, 4, ok, bad, None) == etp.ETP_ERR_INVALID_ARG        # frames misaligned
    assert G(h, 0, None, None, None) == etp.ETP_OK                  # nothing to do
    A = lib.etp_assemble_forces
    assert A(-1, 4, ok, ok, ok, ok, ok, ok, None, None) == etp.ETP_ERR_INVALID_ARG      # N < 0
    assert A(0, 4, ok, ok, ok, ok, ok, ok, None, None) == etp.ETP_ERR_INVALID_ARG       # edges without nodes
    assert A(0, 0, None, None, None, None, None, None, None, None) == etp.ETP_OK        # nothing to do
    assert A(4, 4, ok, ok, ok, ok, ok, None, None, None) == etp.ETP_ERR_INVALID_ARG     # forces NULL
    assert A(4, 4, ok, ok, None, ok, ok, ok, None, None) == etp.ETP_ERR_INVALID_ARG     # rev_perm NULL
    assert A(4, 4, ok, ok, ok, None, ok, ok, ok, None) == etp.ETP_ERR_INVALID_ARG       # virial without r
    assert A(4, 4, ok, ok, ok, ok, ctypes.c_void_p(0x10002), ok, None, None) == etp.ETP_ERR_INVALID_ARG  # grad_r
    rw = ctypes.c_size_t()
    assert lib.etp_radial_workspace_size(h, 100, 8, 64, ctypes.byref(rw)) == etp.ETP_OK and rw.value > 0
    assert lib.etp_radial_workspace_size(h, 100, 33, 64, ctypes.byref(rw)) == etp.ETP_ERR_INVALID_ARG  # n_basis
    assert lib.etp_radial_workspace_size(h, 100, 8, 48, ctypes.byref(rw)) == etp.ETP_ERR_INVALID_ARG   # hidden
    lib.etp_radial_workspace_size(h, 100, 8, 64, ctypes.byref(rw))
    RF, RB = lib.etp_radial_forward, lib.etp_radial_backward
    assert RF(h, 100, 8, 64, 0.0, ok, ok, ok, ok, ok, rw.value, None) == etp.ETP_ERR_INVALID_ARG       # r_cut
    assert RF(h, 100, 8, 64, 5.0, ok, ok, ok, bad, ok, rw.value, None) == etp.ETP_ERR_INVALID_ARG      # w
    assert RF(h, 100, 8, 64, 5.0, ok, ok, ok, ok, ok, rw.value - 1, None) == etp.ETP_ERR_WORKSPACE
    assert RF(h, 0, 8, 64, 5.0, None, None, None, None, None, 0, None) == etp.ETP_OK                  # no edges
    assert RB(h, 100, 8, 64, 5.0, ok, ok, ok, ok, None, ok, ok, ok, rw.value, None) == etp.ETP_ERR_INVALID_ARG
    assert RB(h, 100, 8, 64, 5.0, ok, ok, ok, ok, ok, ok, ok, ok, rw.value - 1, None) == etp.ETP_ERR_WORKSPACE
    sz = ctypes.c_size_t()
    assert lib.etp_reverse_csr_workspace_size(10, 100, ctypes.byref(sz)) == 0 and sz.value > 0
    assert lib.etp_reverse_csr_workspace_size(-1, 100, ctypes.byref(sz)) == etp.ETP_ERR_INVALID_ARG
    R = lib.etp_build_reverse_csr
    assert R(10, 100, ok, ok, ok, ok, ok, ok, sz.value - 1, None) == etp.ETP_ERR_WORKSPACE
    assert R(10, 100, ok, ok, ok, ok, ok, bad, sz.value, None) == etp.ETP_ERR_INVALID_ARG
    assert R(0, 5, ok, ok, ok, ok, ok, ok, sz.value, None) == etp.ETP_ERR_INVALID_ARG
    S = lib.etp_build_reverse_csr_static
    assert S(10, (1 << 18) + 1, ok, ok, ok, ok, ok, None) == etp.ETP_ERR_TOO_LARGE
    assert S((1 << 18) + 1, 10, ok, ok, ok, ok, ok, None) == etp.ETP_ERR_TOO_LARGE
    assert S(10, 100, ok, ok, ctypes.c_void_p(0x10002), ok, ok, None) == etp.ETP_ERR_INVALID_ARG  # rev_ptr
    assert S(-1, 100, ok, ok, ok, ok, ok, None) == etp.ETP_ERR_INVALID_ARG
    ls = ctypes.c_size_t()
    assert lib.etp_locality_schedule_workspace_size(10, 100, ctypes.byref(ls)) == 0 and ls.value > 0
    assert lib.etp_locality_schedule_workspace_size(10, -1, ctypes.byref(ls)) == etp.ETP_ERR_INVALID_ARG
    LS = lib.etp_build_locality_schedule
    full = [ok] * 6
    assert LS(10, 100, ok, ok, ok, 4.5, *full, ok, ls.value - 1, None) == etp.ETP_ERR_WORKSPACE
    assert LS(10, 100, ok, ok, ok, 0.0, *full, ok, ls.value, None) == etp.ETP_ERR_INVALID_ARG      # cell
    assert LS(10, 100, ok, ok, ok, float("nan"), *full, ok, ls.value, None) == etp.ETP_ERR_INVALID_ARG
    assert LS(10, 100, ok, ok, ok, float("inf"), *full, ok, ls.value, None) == etp.ETP_ERR_INVALID_ARG
    assert LS(10, 100, ok, ok, None, 4.5, *full, ok, ls.value, None) == etp.ETP_ERR_INVALID_ARG    # pos
    assert LS(10, 100, ok, ok, ok, 4.5, ok, ok, ok, ok, ok, None, ok, ls.value, None) == etp.ETP_ERR_INVALID_ARG
    assert LS(10, 100, ok, ok, ok, 4.5, *full, ctypes.c_void_p(0x10004), ls.value, None) == etp.ETP_ERR_INVALID_ARG
    assert LS(0, 0, None, None, None, 4.5, *([None] * 6), None, 0, None) == etp.ETP_OK            # nothing to do
    FO, BO = lib.etp_forward_ordered, lib.etp_backward_ordered
    assert FO(h, 4, 4, None, ok, ok, ok, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG    # order NULL
    assert FO(h, 4, 4, ok, ok, None, ok, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG    # ord_edge NULL
    assert FO(h, 4, 4, ok, None, ok, ok, ok, None, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG    # ord_ptr NULL
    assert FO(h, 4, 4, ok, ok, ok, ok, ok, None, ok, ok, bad, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG     # out
    assert BO(h, 4, 4, ok, ok, ok, None, ok, None, ok, ok, ok, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG  # dst
    assert BO(h, 4, 4, None, ok, ok, ok, ok, None, ok, ok, ok, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG  # order
    assert BO(h, 4, 4, ok, ok, ok, ok, ok, None, ok, ok, bad, ok, ok, ok, ok, 1 << 30, None) == etp.ETP_ERR_INVALID_ARG   # grad_out
    assert BO(h, 4, 4, ok, ok, ok, ok, ok, None, ok, ok, ok, None, None, None, ok, 1 << 30, None) == etp.ETP_OK          # nothing
    NP = lib.etp_node_product
    assert NP(None, 4, 2, 0, ok, ok, ok, None) == etp.ETP_ERR_INVALID_ARG      # no plan
    assert NP(h, -1, 2, 0, ok, ok, ok, None) == etp.ETP_ERR_INVALID_ARG        # N < 0
    assert NP(h, 4, 0, 0, ok, ok, ok, None) == etp.ETP_ERR_INVALID_ARG         # K < 1
    assert NP(h, 4, 2, 2, ok, ok, ok, None) == etp.ETP_ERR_INVALID_ARG         # cartesian not 0 / 1
    assert NP(h, 4, 2, 0, None, ok, ok, None) == etp.ETP_ERR_INVALID_ARG       # x NULL
    assert NP(h, 4, 2, 0, ok, None, ok, None) == etp.ETP_ERR_INVALID_ARG       # w NULL with K > 1
    assert NP(h, 4, 2, 1, ok, bad, ok, None) == etp.ETP_ERR_INVALID_ARG        # w misaligned
    assert NP(h, 4, 1, 0, ok, None, bad, None) == etp.ETP_ERR_INVALID_ARG      # out misaligned
    assert NP(h, 0, 3, 1, None, None, None, None) == etp.ETP_OK                # nothing to do
    n = ctypes.c_int()
    assert lib.etp_node_product_ops(None, 0, ctypes.byref(n)) == etp.ETP_ERR_INVALID_ARG
    assert lib.etp_node_product_ops(h, 3, ctypes.byref(n)) == etp.ETP_ERR_INVALID_ARG
    assert lib.etp_node_product_ops(h, 0, None) == etp.ETP_ERR_INVALID_ARG
    V = lib.etp_validate_csr
    assert V(10, 100, None, ok, ok, None) == etp.ETP_ERR_INVALID_ARG
    assert V(10, 100, ok, ok, None, None) == etp.ETP_ERR_INVALID_ARG
    assert lib.etp_plan_destroy(h) == 0
    assert lib.etp_plan_destroy(None) == 0
    assert lib.etp_device_fault(None) == etp.ETP_ERR_INVALID_ARG
    for s in range(8):
        assert lib.etp_status_string(s)
    assert lib.etp_status_string(99) == b"unknown status"


def test_binding_refuses_cpu_tensors(lib):
    import torch

    plan = etp.Plan("0..1", 1, "0..1", 8)
    row_ptr = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(ValueError):
        etp.forward(plan, row_ptr, torch.zeros(0, dtype=torch.int32), torch.zeros(0, 3),
                    torch.zeros(2, 4, 8), torch.zeros(0, 5, 8), out=torch.zeros(2, 4, 8))


def test_binding_checks_dtypes_and_shapes(lib):
    """Wrong dtypes or shapes are refused before anything reaches the library."""
    import torch

    plan = etp.Plan("0..1", 1, "0..1", 8)
    N, E = 3, 4
    row_ptr = torch.tensor([0, 1, 3, 4], dtype=torch.int32)
    src = torch.zeros(E, dtype=torch.int32)
    r, x, w = torch.zeros(E, 3), torch.zeros(N, 4, 8), torch.zeros(E, 5, 8)
    out = torch.zeros(N, 4, 8)
    cases = [dict(x=x.double()), dict(w=torch.zeros(E, 4, 8)), dict(r=torch.zeros(E, 2)),
             dict(src=src.long()), dict(row_ptr=row_ptr[:3]), dict(out=torch.zeros(N, 4, 4))]
    for bad in cases:
        args = dict(row_ptr=row_ptr, src=src, r=r, x=x, w=w, out=out)
        args.update(bad)
        with pytest.raises(ValueError, match="expected"):
            etp.forward(plan, args["row_ptr"], args["src"], args["r"], args["x"], args["w"], out=args["out"])
    with pytest.raises(ValueError, match="expected"):
        etp.edge_frames(plan, torch.zeros(E, 3, dtype=torch.float16))
    with pytest.raises(ValueError, match="expected"):
        etp.assemble_forces(N, row_ptr, row_ptr, src, torch.zeros(E, 3), forces=torch.zeros(N, 2))
    with pytest.raises(ValueError, match="expected"):
        etp.build_reverse_csr(N, row_ptr.long(), src)
    nplan = etp.Plan("0..1", 1, "0..1", 8)
    xn, wn = torch.zeros(N, 4, 8), torch.zeros(2, nplan.n_paths, 8)
    with pytest.raises(ValueError, match="expected"):
        etp.node_product(nplan, xn, torch.zeros(2, 4, 8))
    with pytest.raises(ValueError, match="overlap"):
        etp.node_product(nplan, xn, wn, out=xn)
    with pytest.raises(ValueError, match="required"):
        etp.node_product(nplan, xn, None, K=3)
    with pytest.raises(ValueError, match="CUDA"):
        etp.node_product(nplan, xn, wn)


def test_fused_workspace_size_and_refusals(lib):
    """The fused radial tensor product takes the tensor-core MLP shape only (8 Bessel
    functions, hidden 64); its workspace size is answered on the host."""
    plan = etp.Plan("0..3", 3, "0..3", 128)
    assert etp.fused_workspace_size(plan, 131072) > 0
    with pytest.raises(etp.EtpError) as e:
        etp.fused_workspace_size(plan, 100, n_basis=6, hidden=64)
    assert e.value.status == etp.ETP_ERR_UNSUPPORTED
    with pytest.raises(etp.EtpError):
        etp.fused_workspace_size(plan, 100, n_basis=8, hidden=128)


def test_frames_advised_by_size(lib):
    """Frame records pay while they stay small enough for L2; never at L <= 1."""
    assert etp.Plan("0..3", 3, "0..3", 128).frames_advised(131072)          # 46 MB of records
    assert not etp.Plan("0..3", 3, "0..3", 64).frames_advised(1250256)     # 440 MB
    assert not etp.Plan("0..1", 1, "0..1", 8).frames_advised(256)


@pytest.mark.parametrize("L,o3", [(1, False), (2, True), (3, False), (3, True)])
def test_node_product_ops_count(lib, L, o3):
    """The kernel's cost model: one multiply per operand product that some path uses, one
    FMA per coupling coefficient, one FMA per weighted output component; counted here from
    the oracle's own couplings (nonzero real CG entries; nonzero Cartesian coefficients in
    the independent STF components), which also pins the sparsity of the compiled tables."""
    irreps = "+".join(f"{l}{'e' if l % 2 == 0 else 'o'}" for l in range(L + 1)) if o3 else f"0..{L}"
    plan = etp.Plan(irreps, L, irreps, 8)
    from oracle import nodelocal

    nps = nodelocal.node_paths(irreps)
    terms = sum(int(np.count_nonzero(cg.real_cg(*p))) for p in nps)
    pairs = set()
    for p in nps:
        for a, b, _ in np.argwhere(cg.real_cg(*p) != 0):
            pairs.add((p[0], p[1], int(a), int(b)))
    outs = sum(2 * p[2] + 1 for p in nps)
    assert etp.node_product_ops(plan, False) == len(pairs) + terms + outs
    # Cartesian: the same count from the oracle's Cartesian couplings in independent components
    from cart_layout import coupling_table

    terms, pairs = 0, set()
    for p in nps:
        nz = np.argwhere(np.abs(coupling_table(*p)) > 1e-12)
        terms += len(nz)
        pairs.update((p[0], p[1], int(a), int(b)) for a, b, _ in nz)
    assert etp.node_product_ops(plan, True) == len(pairs) + terms + outs
