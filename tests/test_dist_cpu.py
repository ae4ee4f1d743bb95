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


def _dp_worker(rank, world, port, q):
    """Data-parallel exchange steps of the layer (grouped_gemm_fp32_b200.layer.dp_*) on
    gloo: the whole batch's expert loads, the bias step they drive, the gradient sum."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    import oracle
    from grouped_gemm_fp32_b200 import layer
    w, r, _ = bench.dist_setup(types.SimpleNamespace(impl="reference"))  # gloo
    wl, inp = bench.workload("tiny")
    mine = bench.rank_shard(wl, inp, r)
    dm = wl.dims
    logits = oracle.gate_logits(mine["x"], mine["wg"])
    _, idx, _, _ = oracle.route(logits, mine["bias"], dm.k)
    counts = torch.from_numpy(np.bincount(idx.ravel(), minlength=dm.E).astype(np.int32))
    before = counts.clone()
    total = layer.dp_load_counts(counts)
    every = [None] * w
    dist.all_gather_object(every, idx)
    whole = np.concatenate(every, axis=0)
    # the bias step on the summed loads with the whole batch's token count, as the
    # kernel applies it (bias + gamma * sign(T_all k - load E)), against the oracle's
    # step on the concatenated batch
    import grouped_gemm_fp32_b200 as moe
    gdims = layer.dp_dims(moe.MoeDims.of(dm.T, dm.d, dm.E, dm.k, dm.S, dm.I, dm.P), w)
    gamma = float(np.float32(1e-3))  # the step speed is an f32 on both sides
    diff = gdims.T * dm.k - total.numpy().astype(np.int64) * dm.E
    step = mine["bias"].astype(np.float64) + gamma * np.sign(diff)
    ref = oracle.bias_update(whole, dm.E, mine["bias"], gamma)
    g = torch.full((3, 4), float(rank + 1))
    layer.dp_allreduce_grads([g])
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, torch.equal(counts, before), total.numpy().tolist(),
           np.bincount(whole.ravel(), minlength=dm.E).tolist(), int(gdims.T),
           float(np.abs(step - ref).max()), g.numpy().tolist()))


def test_data_parallel_loads_bias_step_and_gradient_sum():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, untouched, total, whole_counts, T_all, step_err, g in out:
        assert untouched                       # the rank's own counts stay as they were
        assert total == whole_counts           # loads of the concatenated batch
        assert T_all == 2 * 64                 # tiny workload: 64 tokens per rank
        assert step_err == 0.0                 # the sign step on the whole batch's loads
        assert g == [[3.0] * 4] * 3            # 1 + 2, on every rank


def _ep_worker(rank, world, port, q):
    """Expert-parallel exchange (grouped_gemm_fp32_b200.ep) on gloo with CPU tensors:
    counts all-to-all, dispatch of padded segments to their owners (expert-major), and
    the return of the owners' rows into each source's permuted layout."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from grouped_gemm_fp32_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world)
    E, P, d = 6 * world, 8, 4
    El = E // world
    rng = np.random.default_rng(100 + rank)
    counts = rng.integers(0, 20, size=E).astype(np.int32)
    counts[rank] = 0                                   # some empty segments
    ct = torch.from_numpy(counts)
    counts_in = torch.empty_like(ct)
    dist.all_to_all_single(counts_in, ct)
    plan = ep.EPPlan(counts, counts_in.numpy(), rank, world, P)
    # permuted rows: row i of expert g's segment holds (rank, g, i), pad rows -1
    x_perm = torch.full((plan.send_rows, d), -1.0)
    for o, e, a, n in plan.to_owner:
        g = o * El + e
        for i in range(counts[g]):
            x_perm[a + i] = torch.tensor([rank, g, i, 0.0])
    x_recv = torch.full((plan.recv_rows, d), -7.0)
    ep.exchange(*ep.dispatch_lists(plan, x_perm, x_recv), rank)
    ok_dispatch = True
    for s, e, a, n in plan.from_source:
        c = int(counts_in.view(world, El)[s, e])
        for i in range(n):
            want = [s, rank * El + e, i, 0.0] if i < c else [-1.0] * 4
            ok_dispatch &= x_recv[a + i].tolist() == want
    # the owner's "expert" marks each row; the source must get its rows back in place
    y_loc = x_recv.clone()
    y_loc[:, 3] = 100.0 + rank
    y_full = torch.full((plan.send_rows, d), -9.0)
    ep.exchange(*ep.return_lists(plan, y_loc, y_full), rank)
    ok_return = True
    for o, e, a, n in plan.to_owner:
        g = o * El + e
        for i in range(n):
            want = ([rank, g, i] if i < counts[g] else [-1.0] * 3) + [100.0 + o]
            ok_return &= y_full[a + i].tolist() == want
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ok_dispatch, ok_return, plan.recv_rows, int(plan.local_counts.sum())))


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_exchange_moves_segments_both_ways(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_dispatch, ok_return, recv_rows, local_rows in out:
        assert ok_dispatch, rank
        assert ok_return, rank
        assert recv_rows == local_rows


def _cap_worker(rank, world, port, q):
    """ep.check_capacity on gloo: one rank over its receive capacity makes every rank raise."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from grouped_gemm_fp32_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ep.check_capacity(40 + rank, 100)          # everyone within capacity: no error
    raised = False
    try:
        ep.check_capacity(120 if rank == 1 else 10, 100)
    except RuntimeError:
        raised = True
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, raised))


def test_expert_parallel_capacity_overflow_raises_on_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cap_worker, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(raised for _, raised in out)
