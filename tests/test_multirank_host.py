"""The multi-GPU path's host logic under two gloo ranks on CPU: every rank
gets its own batch (distinct seed, no shared data), the timing reduction is
the max over ranks, whole-job throughput counts all ranks' outputs, and the
reference arm prints from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = workloads.WORKLOADS["small_f32"]
    v, g = workloads.generate(w, B=1, L=16, D=4, seed=bench.rank_seed(w, rank))
    ms = bench.max_over_ranks(10.0 + rank, dist)   # rank 1 is the slow one
    ups, gbs = bench.throughput(1000, world, 5, ms, 12)
    q.put((rank, float(v.sum()), ms, ups, gbs))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, ms0, ups0, gbs0), (r1, s1, ms1, ups1, gbs1) = res
    assert s0 != s1                      # distinct batches per rank
    assert ms0 == ms1 == 11.0            # max over ranks, same on every rank
    assert ups0 == ups1 == pytest.approx(2 * 1000 * 5 / 11e-3)
    assert gbs0 == pytest.approx(2 * 1000 * 5 * 12 / 11e-3 / 1e9)


def test_rank_seeds_and_single_rank_reduction():
    w = workloads.WORKLOADS["small_f32"]
    assert bench.rank_seed(w, 0) == w.seed
    assert len({bench.rank_seed(w, r) for r in range(8)}) == 8
    assert bench.max_over_ranks(3.5, None) == 3.5


def test_reference_arm_prints_on_rank0_only():
    """Under two ranks only rank 0 runs and prints the oracle line."""
    env = dict(os.environ, PYTHONPATH=ROOT)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "1", "--workload", "tiny_f32"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
