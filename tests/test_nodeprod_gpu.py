"""GPU parity of the node-local product (etp_node_product) against the FP64 oracle
(oracle/nodelocal.py), spherical and Cartesian couplings.

Every spec (L = 0..3, with and without parities, C from 4 to 128, orders K = 1..5) on a
ragged node count, full comparison; the configuration the bench times (4096 nodes x 128
channels, L = 3, K = 4) on sampled nodes: the product is node-local, so the oracle on a
subset of nodes is exact for those nodes. Tolerance 1e-5 of the largest reference entry:
each output entry is a sum of at most a few hundred FP32 products per step, each step
rounding relative to its own inputs at about 2^-24 per term, over at most four steps.
Order 1 copies x bit for bit; every run repeats bit for bit (no atomics)."""
import numpy as np
import pytest
import torch

import cg_tensor_products_b200 as etp
from cart_layout import from_full, pick, to_full
from cg_tensor_products_b200 import build as etp_build
from gpu_helpers import FWD_TOL, rel_err
from oracle import nodelocal

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    etp_build.build()


def _irreps(L, o3):
    return "+".join(f"{l}{'e' if l % 2 == 0 else 'o'}" for l in range(L + 1)) if o3 else f"0..{L}"


def _inputs(rng, N, L, C, K, P):
    x = rng.standard_normal((N, (L + 1) ** 2, C)).astype(np.float32)
    w = (rng.standard_normal((K - 1, P, C)) / np.sqrt(P)).astype(np.float32)
    return x, w


def _run(plan, x, w, K, cart):
    xd = torch.from_numpy(x).cuda()
    wd = torch.from_numpy(w).cuda() if K > 1 else None
    out = etp.node_product(plan, xd, wd, K=K, cartesian=cart)
    torch.cuda.synchronize()
    return out


def _reference(x, w, irreps, L, cart, nodes=None):
    if nodes is not None:
        x = x[nodes]
    if not cart:
        return nodelocal.node_product(x.astype(np.float64), w.astype(np.float64), irreps)
    full = nodelocal.node_product_cartesian(to_full(x, L), w.astype(np.float64), irreps)
    return from_full(full, L, pick)


SPECS = [(0, False, 4), (1, False, 8), (1, True, 32), (2, False, 64), (2, True, 16), (3, False, 128),
         (3, True, 8), (3, False, 4)]


@pytest.mark.parametrize("cart", [False, True])
@pytest.mark.parametrize("L,o3,C", SPECS)
@pytest.mark.parametrize("K", [1, 2, 4, 5])
def test_every_spec_ragged(L, o3, C, K, cart):
    rng = np.random.default_rng(L * 100 + C + K + 7 * cart)
    irreps = _irreps(L, o3)
    plan = etp.Plan(irreps, L, irreps, C)
    N = 37
    x, w = _inputs(rng, N, L, C, K, plan.n_paths)
    got = _run(plan, x, w, K, cart)
    ref = _reference(x, w, irreps, L, cart)
    assert rel_err(got, ref) <= FWD_TOL


@pytest.mark.parametrize("cart", [False, True])
def test_bench_configuration_sampled(cart):
    """4096 nodes x 128 channels, L = 3 (34 paths), order 4: the bench's launch."""
    rng = np.random.default_rng(11 + cart)
    plan = etp.Plan("0..3", 3, "0..3", 128)
    N, K = 4096, 4
    x, w = _inputs(rng, N, 3, 128, K, plan.n_paths)
    got = _run(plan, x, w, K, cart).cpu().numpy()
    nodes = np.concatenate([[0, 1, N - 1], rng.choice(N, 125, replace=False)])
    ref = _reference(x, w, "0..3", 3, cart, nodes)
    assert rel_err(got[nodes], ref) <= FWD_TOL


def test_order_one_copies_and_runs_repeat_bitwise():
    rng = np.random.default_rng(3)
    plan = etp.Plan("0..3", 3, "0..3", 64)
    x, w = _inputs(rng, 300, 3, 64, 4, plan.n_paths)
    xd, wd = torch.from_numpy(x).cuda(), torch.from_numpy(w).cuda()
    assert torch.equal(etp.node_product(plan, xd, None, K=1), xd)
    for cart in (False, True):
        a = etp.node_product(plan, xd, wd, cartesian=cart)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            b = etp.node_product(plan, xd, wd, cartesian=cart, stream=s)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        assert torch.equal(a, b)


def test_edge_cases():
    """No nodes (nothing launched), one node, the narrowest channel count; weights that
    switch every path off give zeros from order 2 on."""
    plan = etp.Plan("0..2", 2, "0..2", 4)
    x = torch.zeros((0, 9, 4), device="cuda")
    w = torch.zeros((2, plan.n_paths, 4), device="cuda")
    assert etp.node_product(plan, x, w).shape == (0, 9, 4)
    rng = np.random.default_rng(5)
    x1, w1 = _inputs(rng, 1, 2, 4, 3, plan.n_paths)
    got = _run(plan, x1, w1, 3, False)
    assert rel_err(got, _reference(x1, w1, "0..2", 2, False)) <= FWD_TOL
    z = etp.node_product(plan, torch.from_numpy(x1).cuda(), torch.zeros((2, plan.n_paths, 4), device="cuda"))
    torch.cuda.synchronize()
    assert float(z.abs().max()) == 0.0
