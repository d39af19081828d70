"""The allocation-free reverse-CSR entry point (etp_build_reverse_csr_static).

Callers that cannot allocate device memory where they need the reverse CSR (a
plugin inside a host program that owns the GPU memory budget, or a loop that
must not call cudaMalloc) use this variant: its scratch is a fixed device array
inside the library instead of a caller-supplied workspace. This test calls it
through the C ABI and checks that its output is identical (integer work:
bit-exact) to the workspace entry point's, on two calls in a row, and that sizes
beyond its fixed limit are refused before any launch. It lives in its own file,
collected last, and passes alone in a fresh process as well as after the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import cg_tensor_products_b200 as etp
import workloads
from cg_tensor_products_b200 import build as etp_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    etp_build.build()
    return etp._load()


def _graph(seed, n, e):
    rng = np.random.default_rng(seed)
    row_ptr, src, _ = workloads.csr_from_pairs(n, rng.integers(0, n, e), rng.integers(0, n, e))
    return torch.from_numpy(row_ptr).cuda(), torch.from_numpy(src).cuda()


def _static(lib, n, row_ptr, src):
    e = src.numel()
    rev_ptr = torch.full((n + 1,), -7, dtype=torch.int32, device="cuda")
    rev_perm = torch.full((e,), -7, dtype=torch.int32, device="cuda")
    dst = torch.full((e,), -7, dtype=torch.int32, device="cuda")
    st = lib.etp_build_reverse_csr_static(n, e, ctypes.c_void_p(row_ptr.data_ptr()), ctypes.c_void_p(src.data_ptr()),
                                          ctypes.c_void_p(rev_ptr.data_ptr()), ctypes.c_void_p(rev_perm.data_ptr()),
                                          ctypes.c_void_p(dst.data_ptr()),
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == etp.ETP_OK, lib.etp_status_string(st)
    return rev_ptr, rev_perm, dst


def test_static_scratch_matches_workspace_version_twice(lib):
    # 1024 nodes x 128 edges (the micro-benchmark graph's shape), then a ragged multigraph
    cases = [(1024, *_graph(0, 1024, 131072)), (70001, *_graph(1, 70001, 250000))]
    for n, row_ptr, src in cases:
        ref = etp.build_reverse_csr(n, row_ptr, src)
        got = _static(lib, n, row_ptr, src)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    # and the first graph once more, after the scratch held the second graph's data
    n, row_ptr, src = cases[0]
    ref = etp.build_reverse_csr(n, row_ptr, src)
    got = _static(lib, n, row_ptr, src)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


@pytest.mark.parametrize("n,e,with_dst", [(1, 5, True), (7, 0, True), (300, 4000, False), (1, 1, False)])
def test_static_scratch_small_and_degenerate_graphs(lib, n, e, with_dst):
    """Cases only the fixed-scratch path reaches: one source (every edge has source 0,
    no radix pass), no edges at all, and no dst output requested. Compared bit for bit
    with the oracle's reverse CSR."""
    import oracle

    rng = np.random.default_rng(n * 131 + e)
    row_ptr, src, _ = workloads.csr_from_pairs(n, rng.integers(0, n, e), rng.integers(0, n, e))
    o_rp, o_perm, o_dst = oracle.reverse_csr(n, row_ptr, src)
    d_rp, d_src = torch.from_numpy(row_ptr).cuda(), torch.from_numpy(src).cuda()
    for _ in range(2):
        rev_ptr, rev_perm, dst = etp.build_reverse_csr_static(n, d_rp, d_src, with_dst=with_dst)
        torch.cuda.synchronize()
        assert np.array_equal(rev_ptr.cpu().numpy(), o_rp)
        assert np.array_equal(rev_perm.cpu().numpy(), o_perm)
        if with_dst:
            assert np.array_equal(dst.cpu().numpy(), o_dst)
        else:
            assert dst is None


def test_static_scratch_refuses_sizes_above_its_limit(lib):
    big = etp.STATIC_MAX_EDGES + 1
    st = lib.etp_build_reverse_csr_static(10, big, None, None, None, None, None, None)
    assert st == etp.ETP_ERR_TOO_LARGE
    st = lib.etp_build_reverse_csr_static(etp.STATIC_MAX_NODES + 1, 5, None, None, None, None, None, None)
    assert st == etp.ETP_ERR_TOO_LARGE
