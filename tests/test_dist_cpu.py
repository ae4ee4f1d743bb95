"""The multi-process (N > 1) plumbing of bench.py on CPU: world size 2, gloo.

One process per GPU is how the benchmark scales; on the GPU machine the ranks run
independent replicas of the layer step on their own tokens (data parallel, weak
scaling, no collective inside the step) and the step time is the max over
ranks.  These tests run that host logic without a GPU: the max-over-ranks
reduction and barrier, the per-rank token sharding, and the reference arm under
torchrun, where rank 0 alone prints the JSON line and every rank exits 0.
"""
import json
import os
import socket
import subprocess
import sys
import types

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    w, r, _ = bench.dist_setup(types.SimpleNamespace(impl="reference"))  # gloo
    assert (w, r) == (world, rank)
    mx = bench.dist_max(10.0 + rank, w)
    bench.barrier(w)
    wl, inp = bench.workload("tiny")
    mine = bench.rank_shard(wl, inp, r)
    digest = {k: int(np.asarray(v).view(np.uint8).sum()) for k, v in mine.items()}
    gathered = [None] * w
    dist.all_gather_object(gathered, digest)
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((rank, mx, gathered))


def test_two_gloo_ranks_max_barrier_and_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, gathered in out:
        assert mx == 11.0                          # the max over ranks, seen by every rank
        d0, d1 = gathered
        assert d0["x"] != d1["x"]                  # each rank its own tokens
        for k in ("wg", "bias", "w1", "w2"):       # replicated weights
            assert d0[k] == d1[k], k


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1",
           "--warmup", "0"]
    p = subprocess.run(["timeout", "-k", "30", "300"] + cmd, cwd=ROOT, capture_output=True,
                       text=True)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
