"""Throughput of the edge tensor product (forward + VJP) on B200.

One step = the whole hot path on one batch of synthetic input resident in HBM:
reverse CSR (edges grouped by source) + forward + VJP (grad_x, grad_w, grad_r),
all through the C ABI (libetp.so). Default workload: 1024 nodes x 128
neighbours (131072 edges), L = 3, C = 128, 34 paths, fp32.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line (rank 0). With N > 1 (torchrun, one process per GPU) every
rank runs its own replica of the workload (independent problems, no data-path
collective): weak scaling; the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "edges/s fwd+VJP (L=3, C=128) and achieved HBM GB/s vs roofline on 1 B200"
UNIT = "edges/s"
DESCR = {
    "tiny": "32 nodes, 8 nearest neighbours (256 edges), L=1, C=8",
    "micro_l2": "1024 nodes x 128 neighbours (131072 edges), L=2, C=128, 15 paths",
    "micro_l3": "1024 nodes x 128 neighbours (131072 edges), L=3, C=128, 34 paths",
    "water": "3072-atom water box, r_c = 5 A radius graph, L=2, C=64, 15 paths",
    "large": "32768 atoms at 0.1/A^3, r_c = 4.5 A radius graph, L=3, C=64, 34 paths",
}
KERNEL_SOURCES = ["cg_tensor_products_b200/csrc/etp_frame.cuh", "cg_tensor_products_b200/csrc/etp_device.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="micro_l3", choices=sorted(DESCR))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--nodes", type=int, default=None, help="micro workloads: node count (128 neighbours each)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch every step's kernels one by one (default: the step is captured once into a CUDA "
                         "graph and the timed region replays it; per-kernel times then come from eager steps run "
                         "outside the timed region)")
    ap.add_argument("--radial", action="store_true",
                    help="also time the radial weights (w from |r|: Bessel(8) -> 64 -> SiLU -> P*C) and their VJP, "
                         "outside the step")
    ap.add_argument("--frames", choices=["auto", "on", "off"], default="auto",
                    help="edge frame records: as the plan advises (auto), always, or never (the kernels build "
                         "the frames themselves)")
    ap.add_argument("--schedule", choices=["auto", "on", "off"], default="auto",
                    help="locality schedule (rows in the Morton order of the atom positions, several waves of "
                         "tasks): auto = on for workloads with positions whose node features exceed half of L2")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the timings beside the step: the fused radial-weights forward, the VJP of the VJP "
                         "and the Cartesian edge convolution")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU seconds of the oracle baseline")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic traffic and work (what the method must move / compute)
def algorithmic(wl, P, nnz):
    """Bytes and FLOPs per launch of each kernel, counted from the data the method must touch."""
    N, E, C = wl.N, wl.E, wl.C
    D = (wl.L + 1) ** 2
    node = N * D * C * 4
    fwd_bytes = E * (4 * P * C + 12 + 4) + 2 * node + 4 * (N + 1)
    bwd_bytes = E * (2 * 4 * P * C + 12 + 4 + 4 + 12) + 3 * node + 4 * (N + 1)
    return {"fwd_bytes": fwd_bytes, "bwd_bytes": bwd_bytes}


def flops(L, paths, nnz_total, C, E):
    """FLOPs of the plain sparse-CG contraction of the method, per launch (the
    kernels run a cheaper, equivalent edge-frame schedule; these counts give the
    "equivalent" FLOP rates):
    forward 2C(nnz + sum_p d3) per edge (u_p, then the weighted path sum);
    VJP 2C(2 nnz + 3 sum_p d1) per edge (t_p and dL/dY per coupling entry; w*x,
    grad_x and grad_w per input component)."""
    s1 = sum(2 * p[0] + 1 for p in paths)
    s3 = sum(2 * p[2] + 1 for p in paths)
    fwd = 2 * C * (nnz_total + s3) * E
    bwd = 2 * C * (2 * nnz_total + 3 * s1) * E
    return fwd, bwd


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi samples every 100 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.dev)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"samples": 0, "note": "nvidia-smi unavailable"}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        inside = [p for ts, p in rows if self.t0 is not None and self.t0 - 0.1 <= ts <= self.t1 + 0.1] or \
            [p for _, p in rows]
        if not inside:
            return {"samples": 0}
        sm = [float(p[1]) for p in inside if p[1].replace(".", "").isdigit()]
        smax = [float(p[2]) for p in inside if p[2].replace(".", "").isdigit()]
        reasons = set()
        for p in inside:
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 p[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(inside),
                "power_w_max": max(float(p[3]) for p in inside if p[3].replace(".", "").isdigit())
                if any(p[3].replace(".", "").isdigit() for p in inside) else None}


def physical_gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_hash():
    """Hash of the kernel sources' code (line comments and blank lines dropped, so that documentation edits
    keep a capture valid while any code change invalidates it)."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic(kernel, framed, workload, n_nodes, scheduled=False):
    """DRAM bytes (read + write) per launch from a committed ncu capture of the same
    kernel source and launch, else None. The summaries under profiles/ carry lines
    `traffic: <kernel> framed=<0|1> workload=<name> nodes=<N> source=<hash> bytes=<B>`
    (with `schedule=1` for a launch on a locality schedule)."""
    want = {"kernel": kernel, "framed": str(int(framed)), "workload": workload, "nodes": str(n_nodes),
            "source": kernel_source_hash(), "schedule": "1" if scheduled else None}
    pdir = os.path.join(ROOT, "profiles")
    try:
        names = sorted(os.listdir(pdir))
    except OSError:
        return None
    for name in names:
        if not name.endswith((".md", ".txt")):
            continue
        with open(os.path.join(pdir, name)) as f:
            for line in f:
                line = line.strip().strip("`")
                if not line.startswith("traffic: "):
                    continue
                parts = line[len("traffic: "):].split()
                kv = dict(p.split("=", 1) for p in parts[1:] if "=" in p)
                if parts and parts[0] == kernel and all(kv.get(k) == v for k, v in want.items() if k != "kernel"):
                    return float(kv["bytes"])
    return None


# ---------------------------------------------------------------------------
def _oracle_sample(wl, tp, rows):
    """The oracle's forward and VJP on the sub-graph of the given destination rows (their edges only, every
    other row empty): out of those rows, grad_w and grad_r of their edges, grad_x of every source over them.
    Returns (seconds, edges)."""
    import numpy as np

    edges = np.concatenate([np.arange(wl.row_ptr[i], wl.row_ptr[i + 1]) for i in rows])
    counts = np.zeros(wl.N, dtype=np.int64)
    counts[rows] = np.diff(wl.row_ptr)[rows]
    sub_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    src, r, w = wl.src[edges], wl.r[edges], wl.w[edges]
    t0 = time.perf_counter()
    tp.forward(sub_ptr, src, r, wl.x, w, rows=rows)
    tp.backward(sub_ptr, src, r, wl.x, w, wl.g)
    return time.perf_counter() - t0, len(edges)


def cpu_baseline(wl, seconds):
    """The FP64 oracle, as it stands, on a bounded sample: fwd + VJP of the edges of random rows."""
    import numpy as np

    import oracle

    tp = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C)
    rng = np.random.default_rng(1)
    pick = lambda n: np.sort(rng.choice(wl.N, size=min(n, wl.N), replace=False))
    # the work grows with the sampled edges; size the sample to `seconds` (three samples of a third each)
    dt, ne = _oracle_sample(wl, tp, pick(max(2, wl.N // 64)))
    per_edge = max(dt / max(ne, 1), 1e-9)
    want_edges = (seconds / 3) / per_edge
    n_rows = int(max(2, min(wl.N, want_edges / max(wl.E / max(wl.N, 1), 1))))
    runs = sorted((_oracle_sample(wl, tp, pick(n_rows)) for _ in range(3)), key=lambda t: t[1] / t[0])
    dt, ne = runs[1]
    return {"value": ne / dt, "unit": "edges/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"median of 3 samples, each the {ne} edges of {n_rows} random destination rows: forward of "
                      f"those rows and the VJP (grad_x, grad_w, grad_r) over those edges; FP64 C loops with OpenMP, "
                      f"harmonics of the sampled edges in numpy; {dt:.1f} s each"}


def reference_arm(args):
    """The oracle on the host cores: each step a bounded sample of the workload."""
    import numpy as np

    import oracle
    import workloads

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workloads.make(args.workload)
    oracle.build()
    tp = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C)
    rng = np.random.default_rng(2)

    def step(n_rows):
        rows = np.sort(rng.choice(wl.N, size=n_rows, replace=False))
        return _oracle_sample(wl, tp, rows)[1]

    # a step's time grows with its edges; size each step so that the whole run (warm-up + timed steps) takes
    # about two minutes, and at most 2.5 s a step
    t_a = time.perf_counter()
    ne = step(max(2, min(wl.N, wl.N // 64)))
    per_edge = max((time.perf_counter() - t_a) / max(ne, 1), 1e-9)
    budget = min(2.5, 120.0 / max(args.steps + args.warmup, 1))
    rows_per_step = int(max(1, min(wl.N, budget / per_edge / max(wl.E / max(wl.N, 1), 1))))

    for _ in range(args.warmup):
        step(rows_per_step)
    t0 = time.perf_counter()
    ne = sum(step(rows_per_step) for _ in range(args.steps))
    dt = time.perf_counter() - t0
    value = ne / dt
    cores = oracle.num_threads()
    sample = f"each step: the edges of {rows_per_step} random destination rows of {args.workload} (forward of " \
             f"those rows and the VJP: grad_x, grad_w, grad_r over those edges); FP64 oracle"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {DESCR[args.workload]}", "N": wl.N, "E": wl.E,
                   "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ---------------------------------------------------------------------------
def stream_ptr(stream):
    """A torch stream as the C ABI's stream argument."""
    import ctypes

    return ctypes.c_void_p(stream.cuda_stream)


def _time_ms(fn, stream, reps=10, warm=3):
    import torch

    for _ in range(warm):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def measured_bf16():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def extra_timings(etp, lib, plan, wl, d, rev_ptr, rev_perm, dst, gw, stream, dev, nnz_total):
    """Kernels beside the step, each timed alone (CUDA events, 10 calls after 3 warm-up calls) on the same
    workload, each with its roofline:
      - the fused radial-weights tensor product (w = SiLU(bessel(|r|) W1) W2 produced on the tensor cores and
        consumed in the kernel) against the unfused radial_forward + forward; bound by the tensor cores
        (3 TF32 products per FP32 product of the dense layer, TF32 peak = measured bf16 x 1/2);
      - the VJP of the VJP (all three cotangents), against its algorithmic bytes (HBM);
      - the Cartesian edge convolution (forward and VJP) beside the spherical kernels at equal rank, against
        the same algorithmic bytes (HBM);
      - the node-local product at its own fixed size (node_product_timings), against the FP32 pipes."""
    import numpy as np
    import torch

    P = etp._ptr
    tws = torch.empty(max(etp.tp_workspace_size(plan, wl.N, wl.E, False, dev), 16), dtype=torch.uint8, device=dev)
    sp = stream_ptr(stream)
    N, E, C, Pn = wl.N, wl.E, wl.C, plan.n_paths
    D = (wl.L + 1) ** 2
    node = N * D * C * 4
    hbm, hbm_kind = measured_peaks()
    bf16, bf16_kind = measured_bf16()
    out = {}
    # fused radial weights -> tensor product
    rng = np.random.default_rng(7)
    W1 = wl.W1 if wl.W1 is not None else (rng.standard_normal((8, 64)) / np.sqrt(8)).astype(np.float32)
    W2 = wl.W2 if wl.W2 is not None else (rng.standard_normal((64, Pn * C)) / 8.0).astype(np.float32)
    rc = wl.r_cut or 5.0
    W1d, W2d = torch.from_numpy(W1).to(dev), torch.from_numpy(W2).to(dev)
    fws = torch.empty(max(etp.fused_workspace_size(plan, E), 16), dtype=torch.uint8, device=dev)
    fout = torch.empty((N, D, C), device=dev)
    t_fused = _time_ms(lambda: etp._check(lib.etp_fused_forward(
        plan.handle, N, E, P(d["row_ptr"]), P(d["src"]), P(d["r"]), P(d["x"]), 8, 64, rc, P(W1d), P(W2d), P(fout),
        P(fws), fws.numel(), sp), "fused forward"), stream)
    rws = torch.empty(max(etp.radial_workspace_size(plan, E, 8, 64), 16), dtype=torch.uint8, device=dev)
    w_rad = torch.empty((E, Pn, C), device=dev)
    t_rad = _time_ms(lambda: etp._check(lib.etp_radial_forward(
        plan.handle, E, 8, 64, rc, P(d["r"]), P(W1d), P(W2d), P(w_rad), P(rws), rws.numel(), sp), "radial"), stream)
    out2 = torch.empty_like(fout)
    t_tp = _time_ms(lambda: etp._check(lib.etp_forward(
        plan.handle, N, E, P(d["row_ptr"]), P(d["src"]), P(d["r"]), None, P(d["x"]), P(w_rad), P(out2), P(tws),
        tws.numel(), sp), "forward"), stream)
    tflop = 3 * 2.0 * E * 64 * Pn * C
    del w_rad, rws
    out["fused_radial_forward"] = {
        "ms": t_fused, "unfused_ms": t_rad + t_tp, "unfused_radial_forward_ms": t_rad, "unfused_forward_ms": t_tp,
        "speedup_over_unfused": (t_rad + t_tp) / t_fused,
        "roofline": {"bound": "tensor", "achieved": tflop / (t_fused * 1e9), "peak": bf16 / 2, "unit": "TFLOP/s",
                     "frac": tflop / (t_fused * 1e9) / (bf16 / 2),
                     "peak_source": f"{bf16_kind} bf16 x 1/2 (TF32 nominal ratio)",
                     "work": "3 TF32 products x 2 x E x 64 x P x C (the dense layer; the tensor product on the "
                             "FP32 pipes besides)"},
        "hbm_bytes_per_launch": E * 16 + 2 * node + 4 * (N + 1) + 4 * 64 * (8 + Pn * C)}
    # VJP of the VJP
    ggx = torch.randn((N, D, C), device=dev, generator=torch.Generator(device=dev).manual_seed(1))
    ggw = torch.randn((E, Pn, C), device=dev, generator=torch.Generator(device=dev).manual_seed(2)) / Pn ** 0.5
    ggr = torch.randn((E, 3), device=dev, generator=torch.Generator(device=dev).manual_seed(3))
    o = {k: torch.empty_like(v) for k, v in (("g", d["g"]), ("x", d["x"]), ("r", d["r"]))}
    t_dd = _time_ms(lambda: etp._check(lib.etp_double_backward(
        plan.handle, N, E, P(d["row_ptr"]), P(d["src"]), P(rev_ptr), P(rev_perm), P(dst), P(d["r"]), P(d["x"]),
        P(d["w"]), P(d["g"]), P(ggx), P(ggw), P(ggr), P(o["g"]), P(o["x"]), P(gw), P(o["r"]), P(tws), tws.numel(),
        sp), "double"), stream)
    dd_bytes = E * (3 * 4 * Pn * C + 12 * 3 + 4 * 3) + 5 * node + 4 * 2 * (N + 1)
    # the call allocates nothing: its device memory is its arguments (inputs, cotangents, outputs, graph)
    mem = sum(t.numel() * t.element_size() for t in (d["x"], d["w"], d["g"], d["r"], ggx, ggw, ggr, o["g"], o["x"],
                                                     gw, o["r"], d["row_ptr"], d["src"], rev_ptr, rev_perm, dst, tws))
    out["double_backward"] = {
        "ms": t_dd, "bytes_per_launch": dd_bytes, "GBps": dd_bytes / (t_dd * 1e6),
        "roofline": {"bound": "hbm", "achieved": dd_bytes / (t_dd * 1e6), "peak": hbm, "unit": "GB/s",
                     "frac": dd_bytes / (t_dd * 1e6) / hbm, "peak_source": f"{hbm_kind} (hbm_gbs)"},
        "bytes_note": "w and gg_w read, grad_w written (3 x 4PC per edge), r, gg_r, grad_r and three index "
                      "arrays per edge, x, gg_x, g read and grad_g, grad_x written once per node",
        "device_memory_GB": mem / 1e9,
        "device_memory_note": "the call's arguments, its partial-row workspace included; it allocates nothing "
                              "and keeps no [E, P, C] intermediate besides grad_w"}
    del ggx, ggw, ggr, o
    # Cartesian edge convolution at equal rank
    cout = torch.empty_like(fout)
    cgx = torch.empty_like(d["x"])
    cgr = torch.empty_like(d["r"])
    t_cf = _time_ms(lambda: etp._check(lib.etp_cart_forward(
        plan.handle, N, E, P(d["row_ptr"]), P(d["src"]), P(d["r"]), P(d["x"]), P(d["w"]), P(cout), P(tws),
        tws.numel(), sp), "cart"), stream)
    t_cb = _time_ms(lambda: etp._check(lib.etp_cart_backward(
        plan.handle, N, E, P(d["row_ptr"]), P(d["src"]), P(rev_ptr), P(rev_perm), P(dst), P(d["r"]), P(d["x"]),
        P(d["w"]), P(d["g"]), P(cgx), P(gw), P(cgr), P(tws), tws.numel(), sp), "cart backward"), stream)
    t_sf = _time_ms(lambda: etp._check(lib.etp_forward(
        plan.handle, N, E, P(d["row_ptr"]), P(d["src"]), P(d["r"]), None, P(d["x"]), P(d["w"]), P(out2), P(tws),
        tws.numel(), sp), "forward"), stream)
    t_sb = _time_ms(lambda: etp._check(lib.etp_backward(
        plan.handle, N, E, P(d["row_ptr"]), P(d["src"]), P(rev_ptr), P(rev_perm), P(dst), P(d["r"]), None,
        P(d["x"]), P(d["w"]), P(d["g"]), P(cgx), P(gw), P(cgr), P(tws), tws.numel(), sp), "backward"), stream)
    alg = algorithmic(wl, Pn, nnz_total)
    cart = {}
    for key, t, nb in (("cartesian_forward", t_cf, alg["fwd_bytes"]), ("cartesian_backward", t_cb, alg["bwd_bytes"]),
                       ("spherical_forward", t_sf, alg["fwd_bytes"]), ("spherical_backward", t_sb, alg["bwd_bytes"])):
        cart[key] = {"ms": t, "GBps": nb / (t * 1e6), "frac_of_hbm_peak": nb / (t * 1e6) / hbm}
    cart["note"] = ("equal rank: the same graph, weights and path list; both read the edge vectors (no frame "
                    "records); algorithmic bytes of the spherical step for both")
    out["cartesian_vs_spherical"] = cart
    out["node_product"] = node_product_timings(etp, stream, dev)
    return out


def node_product_timings(etp, stream, dev, N=4096, C=128, L=3, K=4, reps=10, warm=3):
    """The node-local product at the size the pages time it (4096 nodes x 128 channels, rank 3,
    correlation order 4; the path-reduced product, forward), spherical and Cartesian couplings.
    Each launch is timed alone with CUDA events after a 256 MB write that flushes L2 (its 67 MB of
    input and output would otherwise stay resident). Bound by the FP32 pipes: the kernel's own
    operation count (etp_node_product_ops: one multiply per operand product, one FMA per
    coupling coefficient and per weighted output component) over 148 SMs x 128 FP32 lanes at
    the 1965 MHz maximum SM clock."""
    import torch

    plan = etp.Plan(f"0..{L}", L, f"0..{L}", C)
    g = torch.Generator(device=dev).manual_seed(5)
    x = torch.randn((N, (L + 1) ** 2, C), device=dev, generator=g)
    w = torch.randn((K - 1, plan.n_paths, C), device=dev, generator=g) / plan.n_paths ** 0.5
    out = torch.empty_like(x)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peak = 148 * 128 * 1.965e9 / 1e12
    res = {"nodes": N, "channels": C, "rank": L, "order": K, "paths": plan.n_paths,
           "page_ms_path_reduced": 0.40, "page_note": "the pages' time for this size and order, GPU not named: context"}
    with torch.cuda.stream(stream):
        for cart in (False, True):
            fn = lambda: etp.node_product(plan, x, w, K=K, cartesian=cart, out=out, stream=stream)
            for _ in range(warm):
                fn()
            total = 0.0
            for _ in range(reps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                b.synchronize()
                total += a.elapsed_time(b)
            ms = total / reps
            ops = etp.node_product_ops(plan, cart) * N * C * (K - 1)
            res["cartesian" if cart else "spherical"] = {
                "ms": ms, "ops_per_node_channel_step": etp.node_product_ops(plan, cart),
                "roofline": {"bound": "alu", "achieved": ops / (ms * 1e9), "peak": peak, "unit": "Top/s",
                             "frac": ops / (ms * 1e9) / peak,
                             "peak_source": "148 SMs x 128 FP32 lanes x 1965 MHz (FMA or multiply: one op)"},
                "hbm_bytes_per_launch": 2 * N * (L + 1) ** 2 * C * 4 + (K - 1) * plan.n_paths * C * 4}
    del flush
    return res


# ---------------------------------------------------------------------------
def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
        return

    import numpy as np
    import torch

    import cg_tensor_products_b200 as etp
    import workloads
    from cg_tensor_products_b200 import replicas

    rank, world, local_rank = replicas.rank_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    replicas.init(world, dev)

    # every rank works on its own instance of the workload (independent problems, seeded by rank)
    wl = workloads.make(args.workload, seed=rank, n_nodes=args.nodes)
    plan = etp.Plan(wl.irreps, wl.L, wl.irreps, wl.C)
    nnz_total = len(plan.couplings()[1])
    N, E = wl.N, wl.E
    host = {k: torch.from_numpy(np.ascontiguousarray(getattr(wl, k))) for k in ("row_ptr", "src", "r", "x", "w", "g")}
    big_nodes = wl.x.nbytes > 64e6  # node features above half of L2: their gathers miss L2 in id order
    scheduled = (wl.pos is not None and big_nodes) if args.schedule == "auto" else args.schedule == "on"
    if scheduled:
        if wl.pos is None:
            raise SystemExit(f"--schedule on: workload {args.workload} has no atom positions")
        host["pos"] = torch.from_numpy(np.ascontiguousarray(wl.pos))

    def io_buffers():
        """A step's inputs (a device copy of `host`) and outputs."""
        b = {k: v.to(dev) for k, v in host.items()}
        b["out"] = torch.empty((N, plan.dim_out, wl.C), device=dev)
        b["gx"] = torch.empty((N, plan.dim_in, wl.C), device=dev)
        b["gw"] = torch.empty((E, plan.n_paths, wl.C), device=dev)
        b["gr"] = torch.empty((E, 3), device=dev)
        return b

    d = io_buffers()
    out, gx, gw, gr = d["out"], d["gx"], d["gw"], d["gr"]
    rev_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
    rev_perm = torch.empty(E, dtype=torch.int32, device=dev)
    dst = torch.empty(E, dtype=torch.int32, device=dev)
    # one scratch for the graph preprocessing and the partial rows of the segment sums (used in turn on one stream)
    ws_bytes = max(etp.reverse_csr_workspace_size(N, E), etp.tp_workspace_size(plan, N, E, scheduled, dev))
    if scheduled:
        ws_bytes = max(ws_bytes, etp.locality_schedule_workspace_size(N, E))
        sched = etp.Schedule(N, E, torch.empty(N, dtype=torch.int32, device=dev),
                             torch.empty(N + 1, dtype=torch.int32, device=dev),
                             torch.empty(E, dtype=torch.int32, device=dev), rev_ptr, rev_perm, dst)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    framed = plan.frames_advised(E) if args.frames == "auto" else args.frames == "on"
    frames = torch.empty((E, etp.FRAME_FLOATS), device=dev) if framed else None
    lib = etp._load()
    stream = torch.cuda.current_stream()
    sp = stream_ptr(stream)
    P = etp._ptr

    def step(ev=None, b=None, s=None):
        """One pass of the path on the buffers b (default d) and stream s (default the current one); the reverse
        CSR, frames and workspace are shared scratch (every use is ordered on the one compute stream)."""
        b = d if b is None else b
        s = stream if s is None else s
        spp = stream_ptr(s)
        if ev:
            ev[0].record(s)
        if scheduled:
            etp._check(lib.etp_build_locality_schedule(N, E, P(b["row_ptr"]), P(b["src"]), P(b["pos"]),
                                                       float(wl.graph_cutoff), *[P(t) for t in sched.tensors()],
                                                       P(ws), ws.numel(), spp), "locality schedule")
        else:
            etp._check(lib.etp_build_reverse_csr(N, E, P(b["row_ptr"]), P(b["src"]), P(rev_ptr), P(rev_perm),
                                                 P(dst), P(ws), ws.numel(), spp), "reverse csr")
        if ev:
            ev[1].record(s)
        if framed:
            etp._check(lib.etp_edge_frames(plan.handle, E, P(b["r"]), P(frames), spp), "edge frames")
        if ev:
            ev[2].record(s)
        # the forward stays in CSR order: on the schedule it reads fewer bytes but is no faster (it is bound by
        # its arithmetic there), while the VJP gains
        etp._check(lib.etp_forward(plan.handle, N, E, P(b["row_ptr"]), P(b["src"]), P(b["r"]), P(frames),
                                   P(b["x"]), P(b["w"]), P(b["out"]), P(ws), ws.numel(), spp), "forward")
        if ev:
            ev[3].record(s)
        if scheduled:
            etp._check(lib.etp_backward_ordered(plan.handle, N, E, P(sched.order), P(rev_ptr), P(rev_perm), P(dst),
                                                P(b["r"]), P(frames), P(b["x"]), P(b["w"]), P(b["g"]), P(b["gx"]),
                                                P(b["gw"]), P(b["gr"]), P(ws), ws.numel(), spp), "backward (scheduled)")
        else:
            etp._check(lib.etp_backward(plan.handle, N, E, P(b["row_ptr"]), P(b["src"]), P(rev_ptr), P(rev_perm),
                                        P(dst), P(b["r"]), P(frames), P(b["x"]), P(b["w"]), P(b["g"]), P(b["gx"]),
                                        P(b["gw"]), P(b["gr"]), P(ws), ws.numel(), spp), "backward")
        if ev:
            ev[4].record(s)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    graph = None
    if not args.eager:
        # per-kernel times from eager steps (outside the timed region), then one capture of the whole step
        for k in range(K):
            step(evs[k])
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream()
        s_cap.wait_stream(stream)
        with torch.cuda.graph(graph, stream=s_cap):
            step(s=s_cap)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
    sampler = ClockSampler(physical_gpu_index(local_rank))
    sampler.start()
    time.sleep(0.3)
    replicas.barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler.mark("t0")
    t_start.record(stream)
    for k in range(K):
        if graph is not None:
            graph.replay()
        else:
            step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark("t1")
    replicas.barrier(world)
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    rc_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    fr_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / K
    fwd_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / K
    bwd_ms = sum(e[3].elapsed_time(e[4]) for e in evs) / K
    ms_step = replicas.max_over_ranks(total_ms / K, world, dev)  # timing only, not the data path
    value = world * E / (ms_step / 1e3)

    # roofline of the dominant kernel (the VJP)
    alg = algorithmic(wl, plan.n_paths, nnz_total)
    peak, peak_kind = measured_peaks()
    fl_fwd, fl_bwd = flops(wl.L, plan.paths, nnz_total, wl.C, E)
    kern = {"graph_prep": "locality schedule" if scheduled else "reverse CSR",
            "reverse_csr_ms" if not scheduled else "locality_schedule_ms": rc_ms,
            "edge_frames_ms": fr_ms if framed else None,
            "forward_ms": fwd_ms, "backward_ms": bwd_ms,
            "forward_GBps": alg["fwd_bytes"] / (fwd_ms * 1e6), "backward_GBps": alg["bwd_bytes"] / (bwd_ms * 1e6),
            "forward_equiv_TFLOPs": fl_fwd / (fwd_ms * 1e9), "backward_equiv_TFLOPs": fl_bwd / (bwd_ms * 1e9),
            "forward_bytes_per_launch": alg["fwd_bytes"], "backward_bytes_per_launch": alg["bwd_bytes"],
            "forward_sparse_cg_flop_per_launch": fl_fwd, "backward_sparse_cg_flop_per_launch": fl_bwd}
    dom = "backward" if bwd_ms >= fwd_ms else "forward"
    achieved = kern[f"{dom}_GBps"]
    kname = f"etp_{'bwd' if dom == 'backward' else 'fwd'}_frame_kernel"
    roofline = {"bound": "hbm", "kernel": f"{kname} ({'frames given' if framed else 'frames built in the kernel'})",
                "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "peak_source": f"{peak_kind} (hbm_gbs, burst copy)",
                "traffic": recorded_traffic(kname, framed, args.workload, N, scheduled)}
    if scheduled:  # the calls below take the reverse CSR in source-id order
        etp._check(lib.etp_build_reverse_csr(N, E, P(d["row_ptr"]), P(d["src"]), P(rev_ptr), P(rev_perm), P(dst),
                                             P(ws), ws.numel(), sp), "reverse csr")

    # force assembly from grad_r (a separate call, not part of the step): forces and per-atom virials
    forces_t = torch.empty((N, 3), device=dev)
    virial_t = torch.empty((N, 9), device=dev)

    def forces_call():
        etp._check(lib.etp_assemble_forces(N, E, P(d["row_ptr"]), P(rev_ptr), P(rev_perm), P(d["r"]), P(gr),
                                           P(forces_t), P(virial_t), sp), "assemble forces")

    for _ in range(3):
        forces_call()
    fa, fb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fa.record(stream)
    for _ in range(20):
        forces_call()
    fb.record(stream)
    torch.cuda.synchronize()
    f_ms = fa.elapsed_time(fb) / 20
    kern["assemble_forces_ms"] = f_ms
    kern["assemble_forces_GBps"] = (40 * E + 48 * N + 8) / (f_ms * 1e6)

    if args.radial:
        rng = np.random.default_rng(99)
        nb, hid, rc = 8, 64, 5.0
        W1 = torch.from_numpy((rng.standard_normal((nb, hid)) / np.sqrt(nb)).astype(np.float32)).to(dev)
        W2 = torch.from_numpy((rng.standard_normal((hid, plan.n_paths * wl.C)) / np.sqrt(hid)).astype(np.float32)).to(dev)
        rws = torch.empty(max(etp.radial_workspace_size(plan, E, nb, hid), 16), dtype=torch.uint8, device=dev)
        w_rad = torch.empty_like(d["w"])
        gW1, gW2 = torch.empty_like(W1), torch.empty_like(W2)
        gr_acc = torch.zeros_like(d["r"])

        def rad_f():
            etp._check(lib.etp_radial_forward(plan.handle, E, nb, hid, rc, P(d["r"]), P(W1), P(W2), P(w_rad), P(rws),
                                              rws.numel(), sp), "radial forward")

        def rad_b():
            etp._check(lib.etp_radial_backward(plan.handle, E, nb, hid, rc, P(d["r"]), P(W1), P(W2), P(gw), P(gW1),
                                               P(gW2), P(gr_acc), P(rws), rws.numel(), sp), "radial backward")

        for fn, key in ((rad_f, "radial_forward_ms"), (rad_b, "radial_backward_ms")):
            for _ in range(3):
                fn()
            ra, rb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ra.record(stream)
            for _ in range(10):
                fn()
            rb.record(stream)
            torch.cuda.synchronize()
            kern[key] = ra.elapsed_time(rb) / 10
        pc = plan.n_paths * wl.C
        kern["radial_forward_TFLOPs"] = 2.0 * E * hid * pc / (kern["radial_forward_ms"] * 1e9)
        kern["radial_backward_TFLOPs"] = 4.0 * E * hid * pc / (kern["radial_backward_ms"] * 1e9)

    # the same kernel against the nominal FP32 rate at the clock seen under load (148 SMs x 128 FMA lanes x 2):
    # the method's sparse-CG FLOP count, which the edge-frame schedule undercuts (it executes fewer)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = (clocks or {}).get("sm_mhz") or (clocks or {}).get("sm_max_mhz") or 1965.0
    fp32_peak = sms * 128 * 2 * mhz * 1e6 / 1e12
    eq = kern[f"{dom}_equiv_TFLOPs"]
    sparse_cg = {"kernel": kname, "equiv_tflops": eq, "nominal_fp32_peak_tflops": fp32_peak,
                 "equiv_over_nominal_peak": eq / fp32_peak,
                 "note": f"NOT an FP32 roofline: the method's plain sparse-CG FLOP count over the kernel time, "
                         f"which the edge-frame schedule undercuts (it executes fewer FLOPs); nominal = {sms} SMs x "
                         f"128 lanes x 2 flop x {mhz:.0f} MHz"}

    extra = None
    if not args.no_extra:
        try:
            extra = extra_timings(etp, lib, plan, wl, d, rev_ptr, rev_perm, dst, gw, stream, dev, nnz_total)
        except Exception as exc:  # reported, not fatal: the step's line stands on its own
            extra = {"error": f"{type(exc).__name__}: {exc}"}

    # end to end through the public API with host buffers (pinned): every step copies its inputs host -> device,
    # runs the path and copies its outputs device -> host, all inside the timed region. Steps are pipelined the
    # way a user streaming batches would run them: two sets of device buffers alternate, the input copies run
    # on one stream, the path on another and the output copies on a third, so step k+1's inputs and step k-1's
    # outputs cross PCIe (both directions at once) while step k computes.
    e2e = None
    if not args.no_e2e:
        pin = {k: v.pin_memory() for k, v in host.items()}
        h_out = {k: torch.empty(d[k].shape).pin_memory() for k in ("out", "gx", "gw", "gr")}
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        d2h = sum(v.numel() * v.element_size() for v in h_out.values())
        k_e2e = max(3, min(K, 20))
        sets = [d, io_buffers()]
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_run(n):
            done_comp, done_out = [], []
            for k in range(n):
                b = sets[k % 2]
                if k >= 2:
                    s_in.wait_event(done_comp[k - 2])   # set b's inputs were read by step k-2
                with torch.cuda.stream(s_in):
                    for key, v in pin.items():
                        b[key].copy_(v, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
                s_comp.wait_event(ready)
                if k >= 2:
                    s_comp.wait_event(done_out[k - 2])  # set b's outputs were read back by step k-2
                step(b=b, s=s_comp)
                c = torch.cuda.Event()
                c.record(s_comp)
                done_comp.append(c)
                s_out.wait_event(c)
                with torch.cuda.stream(s_out):
                    for key, v in h_out.items():
                        v.copy_(b[key], non_blocking=True)
                o = torch.cuda.Event()
                o.record(s_out)
                done_out.append(o)
            return done_out[-1]

        e2e_run(2)
        torch.cuda.synchronize()
        replicas.barrier(world)
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        last = e2e_run(k_e2e)
        s_out.wait_event(last)
        z.record(s_out)
        torch.cuda.synchronize()
        e_ms = replicas.max_over_ranks(a.elapsed_time(z) / k_e2e, world, dev)
        e2e = {"value": world * E / (e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms, "steps": k_e2e,
               "pipelining": "double-buffered: input copies, compute and output copies on three streams"}

    # kernels launched per step: the reverse CSR (one counting pass: counts, chunk scan, chunk-total scan,
    # scatter, edge rows; otherwise counts, scan, edge rows and 4 per 8-bit radix pass: histograms, column scan,
    # digit totals, scatter), frames, forward and backward with their row-combine passes
    n_tiles = (E + 1023) // 1024
    if E > 0 and 1 <= N <= 8192 and (N + 1) * n_tiles <= (1 << 22):
        rc_launches = 5
    else:
        passes = 0
        while (1 << (8 * passes)) < N and passes < 4:
            passes += 1
        rc_launches = (1 if E > 0 else 0) + 1 + (1 if E > 0 else 0) + ((1 if passes == 0 else 4 * passes) if E > 0 else 0)
    if scheduled:  # bounding box (2), Morton keys, 4 radix passes of 4; rank, degrees, scan (3); edge rows,
        # positions, source ranks (3 with edges); then the reverse CSR over the ranks
        rc_launches = 3 + 16 + 3 + ((3 + rc_launches - 1) if E > 0 else 0)  # (its own edge-rows launch is skipped)
    launches = K * (rc_launches + 4 + (1 if framed and E > 0 else 0))  # in the timed steps

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)

    replicas.finalize(world)
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"{args.workload}: {DESCR[args.workload]}" + (f" (reduced to {N} nodes)" if args.nodes else ""),
                   "N": N, "E": E, "L": wl.L, "C": wl.C,
                   "P": plan.n_paths, "cg_nnz": nnz_total,
                   "step": (("locality schedule (Morton order of the positions, ordered CSRs) + " if scheduled
                             else "reverse CSR + ") + ("edge frames + " if framed else "") +
                            ("forward in CSR order + VJP on the schedule: " if scheduled else "") +
                            "forward + VJP (grad_x, grad_w, grad_r), inputs resident in HBM"),
                   "l2": f"inputs larger than L2 (w = {wl.w.nbytes / 1e9:.2f} GB streamed per pass)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "launch": "stream launches" if args.eager else "one CUDA graph replay per step"},
        "roofline": roofline, "sparse_cg_equiv": sparse_cg, "kernels": kern, "beside_the_step": extra, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
        "clocks": clocks,
    }), flush=True)


if __name__ == "__main__":
    main()
