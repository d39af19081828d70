"""GPU parity of the radial weights (etp_radial_forward / etp_radial_backward)
against the FP64 oracle, and of the whole force chain: radial weights -> tensor
product -> VJP -> radial VJP -> assembled forces."""
import numpy as np
import pytest
import torch

import cg_tensor_products_b200 as etp
import oracle
import workloads
from cg_tensor_products_b200 import build as etp_build
from gpu_helpers import FWD_TOL, VJP_TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    etp_build.build()
    oracle.build()


def _params(seed, P, C, nb=8, hidden=64):
    rng = np.random.default_rng(seed)
    W1 = (rng.standard_normal((nb, hidden)) / np.sqrt(nb)).astype(np.float32)
    W2 = (rng.standard_normal((hidden, P * C)) / np.sqrt(hidden)).astype(np.float32)
    return W1, W2, rng


@pytest.mark.parametrize("L,C,nb,hidden,E", [(2, 64, 8, 64, 5000), (3, 128, 8, 64, 3000), (1, 8, 5, 32, 777),
                                             (2, 16, 32, 256, 2000), (3, 32, 8, 64, 1),
                                             (2, 64, 8, 64, 60000), (1, 16, 8, 64, 3001), (2, 32, 8, 64, 129)])
def test_radial_weights_and_vjp_match_oracle(L, C, nb, hidden, E):
    P = workloads.N_PATHS_SO3[L]
    W1, W2, rng = _params(L * 100 + C, P, C, nb, hidden)
    rc = 5.0
    r = (rng.standard_normal((E, 3)) * 2.0).astype(np.float32)
    if E > 10:
        r[3] = 0.0                      # zero length: the basis takes its limit, no derivative
        r[4] = (rc, 0.0, 0.0)           # on the cutoff
    G = rng.standard_normal((E, P, C)).astype(np.float32)
    g0 = rng.standard_normal((E, 3)).astype(np.float32)
    plan = etp.Plan(f"0..{L}", L, f"0..{L}", C)
    d = lambda a: torch.from_numpy(a).cuda()
    w = etp.radial_forward(plan, d(r), d(W1), d(W2), rc)
    grad_r = d(g0.copy())
    gW1, gW2 = etp.radial_backward(plan, d(r), d(W1), d(W2), rc, d(G), grad_r)
    w_b = etp.radial_forward(plan, d(r), d(W1), d(W2), rc)
    grad_r2 = d(g0.copy())
    gW1b, gW2b = etp.radial_backward(plan, d(r), d(W1), d(W2), rc, d(G), grad_r2)
    torch.cuda.synchronize()
    mlp = oracle.radial.RadialMLP(W1, W2, rc, P, C)
    ref_w = mlp.forward(r)
    ref = mlp.backward(r, G)
    assert rel_err(w, ref_w) <= FWD_TOL
    assert rel_err(gW1, ref["grad_W1"]) <= VJP_TOL and rel_err(gW2, ref["grad_W2"]) <= VJP_TOL
    assert rel_err(grad_r - torch.from_numpy(g0).cuda(), ref["grad_r"]) <= VJP_TOL     # accumulated onto g0
    for a, b in ((w, w_b), (gW1, gW1b), (gW2, gW2b), (grad_r, grad_r2)):
        assert torch.equal(a, b)                                                      # bit for bit


def test_force_chain_matches_oracle():
    """Water graph: forces from grad_r through the harmonics plus grad_r through the
    radial weights, all on the GPU, against the same chain in FP64."""
    wl = workloads.make("water")
    P, C, L = wl.P, wl.C, wl.L
    W1, W2, _ = _params(5, P, C)
    rc = 5.0
    plan = etp.Plan(wl.irreps, L, wl.irreps, C)
    t = {k: torch.from_numpy(np.ascontiguousarray(getattr(wl, k))).cuda() for k in ("row_ptr", "src", "r", "x", "g")}
    W1d, W2d = torch.from_numpy(W1).cuda(), torch.from_numpy(W2).cuda()
    w = etp.radial_forward(plan, t["r"], W1d, W2d, rc)
    frames = etp.edge_frames(plan, t["r"])
    out = etp.forward(plan, t["row_ptr"], t["src"], None, t["x"], w, frames=frames)
    rp, perm, dst = etp.build_reverse_csr(wl.N, t["row_ptr"], t["src"])
    gx, gw, gr = etp.backward(plan, t["row_ptr"], t["src"], rp, perm, dst, None, t["x"], w, t["g"], frames=frames)
    gW1, gW2 = etp.radial_backward(plan, t["r"], W1d, W2d, rc, gw, gr)
    F, V = etp.assemble_forces(wl.N, t["row_ptr"], rp, perm, gr, r=t["r"])
    torch.cuda.synchronize()
    assert etp.device_fault() == 0
    mlp = oracle.radial.RadialMLP(W1, W2, rc, P, C)
    tp = oracle.OracleTP(wl.irreps, L, wl.irreps, C)
    w_ref = mlp.forward(wl.r)                                  # FP64 weights: the whole chain in FP64
    x64, g64 = wl.x.astype(np.float64), wl.g.astype(np.float64)
    out_ref = tp.forward(wl.row_ptr, wl.src, wl.r, x64, w_ref)
    vjp = tp.backward(wl.row_ptr, wl.src, wl.r, x64, w_ref, g64)
    rad = mlp.backward(wl.r, vjp["grad_w"])
    g_total = vjp["grad_r"] + rad["grad_r"]
    F_ref, V_ref = oracle.assemble_forces(wl.N, wl.row_ptr, wl.src, wl.r, g_total)
    assert rel_err(out, out_ref) <= FWD_TOL
    for got, want in ((gx, vjp["grad_x"]), (gr, g_total), (gW1, rad["grad_W1"]), (gW2, rad["grad_W2"]),
                      (F, F_ref), (V, V_ref)):
        assert rel_err(got, want) <= VJP_TOL
