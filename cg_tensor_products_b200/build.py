"""Build the CUDA library libetp.so in-tree for sm_100a.

Steps: compile and run the coupling-table generator (csrc/gen_tables.cpp) into
csrc/generated/etp_tables.h, compile every CUDA translation unit with nvcc
(-gencode arch=compute_100a,code=sm_100a), link one shared library next to this
file. Rebuilds only when a source is newer than the library.

    python -m cg_tensor_products_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
GEN_DIR = os.path.join(CSRC, "generated")
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libetp.so")
HEADER = os.path.join(ROOT, "include", "etp.h")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "--expt-relaxed-constexpr", "-lineinfo", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-fvisibility=hidden", "-I" + CSRC, "-I" + os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libetp.so")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cpp")) + [HEADER])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in _sources())


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"command failed ({res.returncode}): {' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    return res.stdout + res.stderr


def generate_tables(verbose=False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    os.makedirs(GEN_DIR, exist_ok=True)
    gen = os.path.join(BUILD_DIR, "gen_tables")
    _run(["g++", "-O2", "-std=c++17", os.path.join(CSRC, "gen_tables.cpp"), "-o", gen], verbose)
    out = os.path.join(GEN_DIR, "etp_tables.h")
    tmp = out + ".tmp"
    _run([gen, tmp], verbose)
    os.replace(tmp, out)
    return out


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Build libetp.so if needed; returns its path."""
    if not force and up_to_date():
        return LIB
    nvcc = _nvcc()
    generate_tables(verbose)
    jobs = []
    for L in range(4):
        jobs.append((os.path.join(CSRC, "etp_kernels_inst.cu"), os.path.join(BUILD_DIR, f"etp_kernels_l{L}.o"),
                     [f"-DETP_L={L}"]))
    for name in ("etp_graph", "etp_forces", "etp_radial", "etp_radial_tc", "etp_fused", "etp_double", "etp_cart", "etp_nodeprod", "etp_api",
                 "etp_static_scratch", "etp_launch"):
        jobs.append((os.path.join(CSRC, name + ".cu"), os.path.join(BUILD_DIR, name + ".o"), []))
    extra = ["-Xptxas", "-v"] if ptxas_info else []

    def compile_one(job):
        src, obj, defs = job
        return _run([nvcc, *ARCH, *NVCC_FLAGS, *extra, *defs, "-c", src, "-o", obj], verbose)

    logs = []
    with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
        for log in ex.map(compile_one, jobs):
            logs.append(log)
    if ptxas_info:
        print("\n".join(logs))
    tmp = LIB + f".tmp{os.getpid()}"
    _run([nvcc, *ARCH, "-shared", "-o", tmp, *[j[1] for j in jobs]], verbose)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills per kernel")
    args = ap.parse_args(argv)
    print(build(force=args.force or args.ptxas_info, verbose=args.verbose, ptxas_info=args.ptxas_info))


if __name__ == "__main__":
    sys.exit(main())
