"""Multi-rank plumbing of the benchmark on CPU (gloo, world size 2).

The hot path shards by batch row with no data-path collective: every rank runs its own
independent batch, and the only cross-rank operations are the barrier around the timed
region and the max-over-ranks reduction of its duration.  These tests cover that host logic
and the reference arm under a two-rank launch.
"""

import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import workloads

    ms = bench.max_over_ranks(10.0 * (rank + 1), dist, torch.device("cpu"))
    rows = list(workloads.shard_rows(13, world, rank))
    all_rows = [None] * world
    dist.all_gather_object(all_rows, rows)
    dist.barrier()
    q.put((rank, ms, all_rows))
    dist.destroy_process_group()


def test_two_rank_max_timing_and_row_sharding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, all_rows in out:
        assert ms == 20.0  # both ranks see the slowest rank's time
        flat = [r for part in all_rows for r in part]
        assert flat == list(range(13))  # contiguous, disjoint, complete


def test_shard_rows_balanced():
    import workloads

    for total in (0, 1, 7, 64, 65):
        for world in (1, 2, 3, 8):
            parts = [list(workloads.shard_rows(total, world, r)) for r in range(world)]
            assert sum(parts, []) == list(range(total))
            sizes = [len(x) for x in parts]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="CPU (gloo) launch of the reference arm")
def test_reference_arm_two_ranks_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    import json

    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
