"""The benchmark's own bookkeeping, without a GPU: the algorithmic bytes behind the
roofline, the lookup of recorded DRAM traffic, and the default timing settings."""
import sys

import bench
import workloads


def test_algorithmic_bytes_of_the_benchmark_workload():
    """Forward: w, r, src per edge + x and out per node + row_ptr; VJP: w read and
    grad_w written, r, src, rev_perm, dst, grad_r per edge + x, grad_out, grad_x per
    node + row_ptr (fp32 data, int32 indices)."""
    class Shape:   # micro_l3's sizes without generating it
        N, E, C, L = 1024, 131072, 128, 3
    alg = bench.algorithmic(Shape, 34, 611)
    assert alg["fwd_bytes"] == 131072 * (4 * 34 * 128 + 16) + 2 * 1024 * 16 * 128 * 4 + 4 * 1025 == 2300579844
    assert alg["bwd_bytes"] == 131072 * (8 * 34 * 128 + 32) + 3 * 1024 * 16 * 128 * 4 + 4 * 1025 == 4592766980


def test_recorded_traffic_only_for_its_own_kernel_code_and_workload():
    got = bench.recorded_traffic("etp_bwd_frame_kernel", True, "micro_l3", 1024)
    assert got is None or 0.99 < got / 4592766980 < 1.02     # within the committed record's measured ratio
    assert bench.recorded_traffic("etp_bwd_frame_kernel", True, "large", 32768) is None
    assert bench.recorded_traffic("etp_bwd_frame_kernel", False, "micro_l3", 1024) is None
    assert bench.recorded_traffic("etp_bwd_frame_kernel", True, "micro_l3", 600) is None


def test_kernel_source_hash_ignores_comments(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_text("int a; // one\n\nint b;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ["k.cuh"])
    h1 = bench.kernel_source_hash()
    src.write_text("int a; // another comment\nint b;   \n// and a line of comment only\n")
    assert bench.kernel_source_hash() == h1
    src.write_text("int a; int b;\n")
    assert bench.kernel_source_hash() != h1


def test_default_timing_settings(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    args = bench.parse()
    assert args.gpus == 1 and args.warmup >= 3 and args.steps >= 1 and args.workload == "micro_l3"
    assert not args.eager and args.frames == "auto" and args.impl == "ours"
    assert args.workload in bench.DESCR and set(bench.DESCR) == set(workloads.SPECS)
