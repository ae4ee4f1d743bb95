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
    """Expert parallelism's host side on gloo with CPU tensors: the all-gather of every
    rank's per-expert counts (ep.gather_counts, the only collective the exchange needs)
    and the plan every rank derives from them: what a source writes where must be where
    its owner expects it, for every pair of ranks, including ranks that send an owner
    nothing."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist
    from common import ep_plan_reference
    from grouped_gemm_fp32_b200 import MoeDims, ep
    dist.init_process_group("gloo", rank=rank, world_size=world)
    E, P, k, T = 4 * world, 32, 2, 40
    El = E // world
    eb = ep.EPBuffers(MoeDims.of(T, 64, E, k, 1, 64, P), rank, world, device="cpu")
    rng = np.random.default_rng(100 + rank)
    counts = rng.integers(0, 20, size=E).astype(np.int32)
    counts[rank] = 0                             # an empty segment on every rank
    if rank == 0 and world > 2:
        counts[2 * El:3 * El] = 0                # rank 0 sends owner 2 nothing at all
    eb.full.counts.copy_(torch.from_numpy(counts))
    ep.gather_counts(eb)
    table = eb.counts_all.numpy().copy()
    cap = eb.cap
    plans = [ep_plan_reference(table, r, P, cap) for r in range(world)]
    mine = plans[rank]
    ok = bool(np.array_equal(table[rank], counts))
    # the table is the same on every rank
    allt = [torch.zeros_like(eb.counts_all) for _ in range(world)]
    dist.all_gather(allt, eb.counts_all)
    ok &= all(torch.equal(t, eb.counts_all) for t in allt)
    pad = (table + P - 1) // P * P
    for o in range(world):
        own = plans[o]
        # source `rank`'s segment of each expert of owner o lands where o expects it
        for e in range(El):
            g = o * El + e
            ok &= int(mine["send_dst"][g]) == int(own["recv_row"][rank, e])
            ok &= int(own["recv_cnt"][rank, e]) == int(pad[rank, g])
            ok &= int(own["src_off"][rank, e]) == int(pad[rank, :g].sum())
        # owner o's received segments tile its rows [0, total) in expert-major order
        spans = sorted((int(own["recv_row"][s, e]), int(own["recv_cnt"][s, e]))
                       for e in range(El) for s in range(world))
        pos = 0
        for start, n in spans:
            ok &= start == pos
            pos += n
        ok &= pos == int(own["counts_loc"].sum())
    zero_from_peer = any(pad[s, o * El:(o + 1) * El].sum() == 0
                         for s in range(world) for o in range(world) if s != o)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ok, zero_from_peer, [int(v) for v in mine["over"]]))


@pytest.mark.parametrize("world", [2, 3, 4])
def test_expert_parallel_plan_agrees_across_ranks(world):
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
    for rank, ok, zero_from_peer, over in out:
        assert ok, rank
        assert over == [0] * world
    if world > 2:
        assert any(z for _, _, z, _ in out)  # some rank receives zero rows from a peer


def test_expert_parallel_plan_flags_an_owner_over_capacity():
    # rank 1 is sent more rows than the receive buffers hold: every rank's plan says so
    # (the device kernels then write nothing into that owner's buffers)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from common import ep_plan_reference
    table = np.array([[100, 0, 300, 40], [5, 0, 200, 1]])
    for r in range(2):
        assert ep_plan_reference(table, r, 32, 600)["over"].tolist() == [0, 1]
