"""The C ABI from a plain C program (tests/c_abi/etp_c_caller.c, built with gcc
against include/etp.h and libetp.so): no Python binding involved.

CPU: the program builds, links and passes its host-side checks. GPU: it runs the
reverse CSR, edge frames, forward and VJP on CUDA-runtime buffers, and its
outputs match the FP64 oracle."""
import os
import subprocess

import numpy as np
import pytest

import cg_tensor_products_b200 as etp
import oracle
import workloads
from cg_tensor_products_b200 import build as etp_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def caller(tmp_path_factory):
    if not os.path.exists(etp.LIB_PATH):
        etp_build.build()
    exe = str(tmp_path_factory.mktemp("c_abi") / "etp_c_caller")
    libdir = os.path.dirname(etp.LIB_PATH)
    cmd = ["gcc", "-std=c11", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_abi", "etp_c_caller.c"),
           "-L", libdir, "-letp", f"-Wl,-rpath,{libdir}", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_caller_host_checks(caller):
    res = subprocess.run([caller, "host"], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stderr


@pytest.mark.gpu
@pytest.mark.parametrize("L,o3,C", [(3, False, 16), (2, True, 128), (1, False, 4)])
def test_c_caller_matches_oracle(caller, tmp_path, L, o3, C):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.build()
    irreps = "+".join(f"{l}{'eo'[l % 2]}" for l in range(L + 1)) if o3 else f"0..{L}"
    P = len(oracle.paths.enumerate_paths(irreps, L, irreps))
    wl = workloads.random_graph(np.random.default_rng(40 + L + C), 29, 333, L, C, P)
    src_path, out_path = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(src_path, "wb") as f:
        np.array([wl.N, wl.E, L, C, int(o3)], np.int32).tofile(f)
        for a, t in ((wl.row_ptr, np.int32), (wl.src, np.int32), (wl.r, np.float32), (wl.x, np.float32),
                     (wl.w, np.float32), (wl.g, np.float32)):
            np.ascontiguousarray(a, dtype=t).tofile(f)
    res = subprocess.run([caller, "run", str(src_path), str(out_path)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    D = (L + 1) ** 2
    raw = np.fromfile(out_path, np.uint8)
    off = 0

    def take(n, dt):
        nonlocal off
        a = raw[off:off + 4 * n].view(dt)
        off += 4 * n
        return a

    out = take(wl.N * D * C, np.float32).reshape(wl.N, D, C)
    gx = take(wl.N * D * C, np.float32).reshape(wl.N, D, C)
    gw = take(wl.E * P * C, np.float32).reshape(wl.E, P, C)
    gr = take(wl.E * 3, np.float32).reshape(wl.E, 3)
    rev_ptr, rev_perm = take(wl.N + 1, np.int32), take(wl.E, np.int32)
    forces = take(wl.N * 3, np.float32).reshape(wl.N, 3)
    assert off == raw.size
    tp = oracle.OracleTP(irreps, L, irreps, C)
    ref_out = tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w)
    ref = tp.backward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w, wl.g)

    def rel(a, b):
        return float(np.max(np.abs(a.astype(np.float64) - b)) / max(np.max(np.abs(b)), 1e-300))

    assert rel(out, ref_out) <= 1e-5
    for got, key in ((gx, "grad_x"), (gw, "grad_w"), (gr, "grad_r")):
        assert rel(got, ref[key]) <= 1e-4, key
    o_rp, o_perm, _ = oracle.reverse_csr(wl.N, wl.row_ptr, wl.src)
    assert np.array_equal(rev_ptr, o_rp) and np.array_equal(rev_perm, o_perm)
    F_ref, _ = oracle.assemble_forces(wl.N, wl.row_ptr, wl.src, wl.r, ref["grad_r"])
    assert rel(forces, F_ref) <= 1e-4
