"""The multi-GPU path on CPU: world size 2 over gloo (no GPU needed).

On several GPUs every rank works on its own independent problems and the only
communication is host bookkeeping (a barrier, the max of the ranks' times). These
tests run that bookkeeping with two real processes, each also evaluating its
shard of a set of small independent graphs with the oracle, and check that the
shards together give exactly the single-process results.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from cg_tensor_products_b200 import replicas

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_covers_units_disjointly():
    for n in (0, 1, 7, 64, 1001):
        for world in (1, 2, 3, 8):
            parts = [replicas.shard(n, r, world) for r in range(world)]
            got = [u for p in parts for u in p]
            assert got == list(range(n))
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        replicas.shard(10, 2, 2)


def _problem(k):
    """Independent problem k: a small random graph of the workload family."""
    import workloads

    return workloads.random_graph(np.random.default_rng(1000 + k), 12, 60, 1, 8, 5)


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import oracle

    r, w, lr = replicas.rank_env()
    assert (r, w, lr) == (rank, world, rank)
    dev = torch.device("cpu")
    replicas.init(world, dev, timeout_s=60)
    n_problems = 5
    mine = replicas.shard(n_problems, rank, world)
    results = {}
    for k in mine:
        wl = _problem(k)
        tp = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C)
        results[k] = float(np.abs(tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w)).sum())
    replicas.barrier(world)
    slowest = replicas.max_over_ranks(10.0 + rank, world, dev)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"mine": list(mine), "results": results, "max": slowest}, f)
    replicas.finalize(world)


def test_two_gloo_ranks_share_independent_problems(tmp_path):
    import oracle

    oracle.build()
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert got[0]["max"] == got[1]["max"] == 11.0          # the slowest rank's time, on every rank
    assert sorted(got[0]["mine"] + got[1]["mine"]) == list(range(5))
    merged = {int(k): v for g in got for k, v in g["results"].items()}
    for k in range(5):                                        # same as one process doing everything
        wl = _problem(k)
        tp = oracle.OracleTP(wl.irreps, wl.L, wl.irreps, wl.C)
        assert merged[k] == float(np.abs(tp.forward(wl.row_ptr, wl.src, wl.r, wl.x, wl.w)).sum())


def test_reference_arm_under_torchrun_prints_once():
    """`bench.py --impl reference` launched as 2 ranks: rank 0 alone runs and prints one line."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
